"""GPU parity: csla_indexer_scores (1e-3 relative to max(|oracle|,
1e-3*rowmax)) and csla_topk_select (exact on given fp32 scores; on the
pipeline's scores the set equals the oracle's except inside the 1e-4
ambiguity band around the k-th score)."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from csla_synth import normal, integers
from csla_synth.workloads import CSA_DECODE, CSA_TINY, layer_params, step_inputs
from gpu_helpers import DEV, act_tensor, assert_no_device_error, check_scores, upload_layer
from helpers import oracle_cache

pytestmark = pytest.mark.gpu

GAP_TOL = 1e-4          # top-k ambiguity band


def run_indexer(w, lb, si, p, B, max_len):
    cfg = lb.cfg()
    stride = max_len // w.m
    scores = torch.full((B, stride), float("nan"), dtype=torch.float32, device=DEV)
    ws_bytes = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, max_len)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    cq = act_tensor(w, si["cq"])
    W = act_tensor(w, p["W_iq"])
    hw = torch.as_tensor(si["head_w"], dtype=torch.float32, device=DEV)
    dt = C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32
    C.csla_indexer_scores(cfg, lb.state(), lb.cache(), slots, B, max_len, cq, dt, W, dt, hw, scores, stride,
                          ws, ws_bytes)
    return scores, slots


def oracle_scores(w, cv, s, L, si, p):
    nv = L // w.m
    qI = oracle.index_query(si["cq"][s], p["W_iq"], w.HI, w.dI)
    return oracle.index_scores(qI, si["head_w"][s], cv.gather_keys(s, nv))


@pytest.mark.parametrize("w,lens", [
    (dataclasses.replace(CSA_TINY, B=3, L=2048, name="idx_tiny"), [2048, 515, 3]),
    (dataclasses.replace(CSA_DECODE, B=2, L=5000, name="idx_big"), [5000, 1113]),
])
def test_indexer_matches_oracle(w, lens):
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 3)
    max_len = max(lens)
    scores, _ = run_indexer(w, lb, si, p, len(lens), max_len)
    assert_no_device_error()
    got_all = scores.cpu().numpy()
    for s, L in enumerate(lens):
        nv = L // w.m
        if nv:
            ref = oracle_scores(w, cv, s, L, si, p)
            check_scores(got_all[s, :nv].astype(np.float64), ref)
        assert np.all(np.isnan(got_all[s, nv:])), "entries past the visible range were written"


def _topk_gpu(scores_np, lens_n, k, m=4):
    """Run csla_topk_select on given fp32 scores; lens_n = visible entries per request."""
    B, stride = scores_np.shape
    from compressed_sparse_long_append_b200.layer import LayerBuffers, LayerShape
    lb = LayerBuffers(LayerShape(m=m, D=128, H=8, HI=4, dI=64, dc=128), B, 1, 1, DEV)
    lb.len.copy_(torch.tensor([n * m for n in lens_n], dtype=torch.int32))
    sc = torch.as_tensor(scores_np, dtype=torch.float32, device=DEV)
    idx = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    C.csla_topk_select(lb.cfg(), lb.state(), slots, B, stride * m, sc, stride, k, idx)
    assert_no_device_error()
    return idx.cpu().numpy()


@pytest.mark.parametrize("n,k", [(0, 8), (5, 8), (64, 64), (1000, 64), (32768, 512), (50000, 1024),
                                 (70000, 2048)])
def test_topk_exact_on_given_scores(n, k):
    """Exact comparison on identical fp32 inputs, with heavy ties, signed
    zeros and both the shared-memory and the global-memory key paths."""
    B = 3
    stride = max(n, 1)
    sc = np.zeros((B, stride), np.float32)
    for b in range(B):
        v = normal(b, "topk/%d/%d" % (n, k), (stride,)).astype(np.float32)
        if b == 1:
            v = np.round(v * 4) / 4                      # many exact ties
        if b == 2:
            v = np.where(integers(9, "z/%d" % n, (stride,), 0, 3) == 0, np.float32(-0.0), v)
            v = np.where(integers(9, "z2/%d" % n, (stride,), 0, 3) == 0, np.float32(0.0), v).astype(np.float32)
        sc[b] = v
    got = _topk_gpu(sc, [n] * B, k)
    for b in range(B):
        ref = oracle.topk(sc[b, :n].astype(np.float64), k)
        assert np.array_equal(got[b], ref), (b, got[b][:10], ref[:10])


def test_topk_ragged_batch():
    lens = [40000, 7, 600, 41000]
    k = 512
    stride = max(lens)
    sc = np.stack([normal(5, "rag/%d" % i, (stride,)) for i in range(len(lens))]).astype(np.float32)
    got = _topk_gpu(sc, lens, k)
    for b, n in enumerate(lens):
        assert np.array_equal(got[b], oracle.topk(sc[b, :n].astype(np.float64), k))


def test_pipeline_topk_set_within_ambiguity_band():
    w = dataclasses.replace(CSA_DECODE, B=2, L=12000, name="topk_pipe")
    lens = [12000, 9001]
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 4)
    scores, slots = run_indexer(w, lb, si, p, 2, max(lens))
    idx = torch.full((2, w.k), -7, dtype=torch.int32, device=DEV)
    C.csla_topk_select(lb.cfg(), lb.state(), slots, 2, max(lens), scores, max(lens) // 4, w.k, idx)
    assert_no_device_error()
    got = idx.cpu().numpy()
    for s, L in enumerate(lens):
        ref_scores = oracle_scores(w, cv, s, L, si, p)
        ref = oracle.topk(ref_scores, w.k)
        g = got[s][got[s] >= 0]
        assert np.all(np.diff(g) > 0) and len(g) == min(w.k, L // 4)
        kth = np.sort(ref_scores)[::-1][w.k - 1]
        must = set(np.nonzero(ref_scores > kth + GAP_TOL)[0].tolist())
        never = set(np.nonzero(ref_scores < kth - GAP_TOL)[0].tolist())
        gs = set(g.tolist())
        assert must <= gs and not (gs & never)
        assert len(gs ^ set(ref[ref >= 0].tolist())) <= 2 * len(np.nonzero(np.abs(ref_scores - kth) <= GAP_TOL)[0])


@pytest.mark.parametrize("key_fmt", [0, 1])
def test_indexer_scores_do_not_depend_on_the_batch(key_fmt):
    """One request's scores bit-identical whether it is scored alone or as
    one of 200 rows: the batch changes the projection's tiling (the request
    lands in another 128-row tile and TMEM lane of the tensor-core GEMM) and
    the indexer's grid, never a row's arithmetic."""
    w = dataclasses.replace(CSA_DECODE, B=1, L=3000, key_fmt=key_fmt, name="idx_inv")
    cv, p = oracle_cache(w, [3000])
    lb = upload_layer(w, cv, [3000])
    nb = 200
    # 200 slots that all read the one request's pages
    from compressed_sparse_long_append_b200.layer import LayerBuffers
    from gpu_helpers import fill_layer, shape_of
    big = LayerBuffers(shape_of(w), nb, lb.n_pages, lb.bt_stride, DEV)
    fill_layer(big, w, cv, [3000])
    big.block_table.copy_(lb.block_table.expand(nb, -1))
    big.len.fill_(3000)
    big.win_rows.copy_(lb.win_rows.expand(nb, -1, -1))
    big.win_scales.copy_(lb.win_scales.expand(nb, -1))
    si = step_inputs(dataclasses.replace(w, B=nb), 11)
    rows = [0, 37, 131, 199]
    cq_all = np.stack([si["cq"][r] for r in range(nb)])
    hw_all = np.stack([si["head_w"][r] for r in range(nb)])
    s_big, _ = run_indexer(w, big, {"cq": cq_all, "head_w": hw_all}, p, nb, 3000)
    for r in rows:
        s_one, _ = run_indexer(w, lb, {"cq": cq_all[r:r + 1], "head_w": hw_all[r:r + 1]}, p, 1, 3000)
        nv = 3000 // w.m
        assert torch.equal(s_one[0, :nv].view(torch.int32), s_big[r, :nv].view(torch.int32)), r
    assert_no_device_error()
