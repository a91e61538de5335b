"""Failure detection without a GPU fault: bad inputs that only the device can
see are recorded in the library's device error word and skipped, and a
bounded wait that runs out returns with CSLA_DEVERR_TIMEOUT; in every case
the kernels return and the context stays usable.

  * a block-table entry outside the page pool (injected on the host) ->
    CSLA_DEVERR_PAGE from the indexer and the attention call; the rows of
    that page are skipped, every other request is unaffected bit for bit;
  * csla_check_wait_timeout: the library's bounded mbarrier wait on a
    barrier nobody arrives at, with a 1 ms limit -> CSLA_DEVERR_TIMEOUT, and
    an attention call right after it is correct."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from csla_synth.workloads import CSA_DECODE, step_inputs
from gpu_helpers import DEV, act_tensor, assert_no_device_error, check_out, upload_layer
from helpers import oracle_cache

pytestmark = pytest.mark.gpu

W = dataclasses.replace(CSA_DECODE, B=3, L=3000, k=64, name="failures")


def _run(w, lb, si, p, lens, idx=None):
    """Indexer, top-k (when idx is None) and attention for all requests."""
    B, ml = len(lens), max(lens)
    cfg = lb.cfg()
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    stride = ml // w.m
    scores = torch.full((B, stride), float("nan"), dtype=torch.float32, device=DEV)
    wsb = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, ml)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    C.csla_indexer_scores(cfg, lb.state(), lb.cache(), slots, B, ml, act_tensor(w, si["cq"][:B]), C.CSLA_BF16,
                          act_tensor(w, p["W_iq"]), C.CSLA_BF16,
                          torch.as_tensor(si["head_w"][:B], dtype=torch.float32, device=DEV), scores, stride, ws, wsb)
    if idx is None:
        idx = torch.zeros((B, w.k), dtype=torch.int32, device=DEV)
        C.csla_topk_select(cfg, lb.state(), slots, B, ml, scores, stride, w.k, idx)
    out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.float32, device=DEV)
    wsa = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, B, w.k)
    wa = torch.zeros(wsa, dtype=torch.uint8, device=DEV)
    C.csla_csa_attend(cfg, lb.state(), lb.cache(), slots, B, act_tensor(w, si["q"][:B]), C.CSLA_BF16, idx, w.k,
                      torch.as_tensor(p["sink"], dtype=torch.float32, device=DEV),
                      torch.as_tensor(p["gamma_q"], dtype=torch.float32, device=DEV), out, C.CSLA_F32,
                      C.CSLA_VARIANT_AUTO, wa, wsa)
    return scores, idx, out


def test_block_table_entry_outside_the_pool_is_recorded_and_skipped():
    lens = [3000, 2500, 2800]
    cv, p = oracle_cache(W, lens)
    lb = upload_layer(W, cv, lens)
    si = step_inputs(W, 31)
    clean_scores, clean_idx, clean_out = _run(W, lb, si, p, lens)
    assert_no_device_error()
    # the page holding request 1's first selected entry now names a page past the pool
    epp = 128 // W.m
    bad_col = int(clean_idx[1, 0].item()) // epp
    lb.block_table[1, bad_col] = lb.n_pages + 7
    scores, _, out = _run(W, lb, si, p, lens, idx=clean_idx)
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits == C.CSLA_DEVERR_PAGE, (rc, bits)
    # the other requests: bit-identical scores and outputs
    for s in (0, 2):
        assert torch.equal(torch.nan_to_num(scores[s], nan=-7.0), torch.nan_to_num(clean_scores[s], nan=-7.0))
        assert torch.equal(out[s], clean_out[s])
    # request 1: the bad page's entries are not scored, the rest are as before
    bad = slice(bad_col * epp, (bad_col + 1) * epp)
    s1, c1 = scores[1].cpu().numpy(), clean_scores[1].cpu().numpy()
    assert np.all(np.isnan(s1[bad]))
    keep = np.ones(len(s1), bool)
    keep[bad] = False
    nv = lens[1] // W.m
    keep[nv:] = False
    assert np.array_equal(s1[keep], c1[keep])
    # request 1's attention skips the selected rows on that page: the oracle
    # over the remaining selected rows plus the window
    sel = clean_idx[1].cpu().numpy()
    kept = sel[(sel < bad.start) | (sel >= bad.stop)]
    rows = cv.gather_set(1, lens[1], kept)
    ref, _ = oracle.attend(si["q"][1], p["gamma_q"], lens[1] - 1, rows, p["sink"], W.eps, W.theta, W.d_rope)
    assert len(kept) < len(sel)
    check_out(out[1].cpu().numpy().astype(np.float64), ref)


def test_bounded_wait_runs_out_and_reports_timeout():
    assert C.csla_device_error() == (C.CSLA_OK, 0)
    C.csla_check_wait_timeout(1000)
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits == C.CSLA_DEVERR_TIMEOUT, (rc, bits)
    # the context is usable: a full step right after it is correct
    lens = [1500, 900]
    w = dataclasses.replace(W, B=2, L=1500, name="after_timeout")
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 32)
    _, idx, out = _run(w, lb, si, p, lens)
    assert_no_device_error()
    got = out.cpu().numpy().astype(np.float64)
    for s, L in enumerate(lens):
        rows = cv.gather_set(s, L, idx[s].cpu().numpy())
        ref, _ = oracle.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"], w.eps, w.theta, w.d_rope)
        check_out(got[s], ref)
