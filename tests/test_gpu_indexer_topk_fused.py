"""GPU parity of csla_indexer_topk (the indexer and the top-k in one call,
the scores of long rows never stored) against csla_indexer_scores followed
by csla_topk_select on the same inputs: idx equal, element for element.

The index keys are seeded random values written straight into a scattered
page pool (no compressor run): the selection is what is compared.  The cases
reach every path of the fused call: rows of at most k entries, rows of at
most 6144 entries (every entry a candidate), long rows through the sample
threshold, and rows that fall back to the stored-score path (all scores
equal: more candidates than the call keeps), with bf16 and E4M3 keys, query
rows of one request (several rows per key tile) and decode rows of several
requests.  A few rows are also checked against the oracle's top-k of the
two-call path's scores."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import LayerBuffers
from csla_synth import torch_gen as TG
from csla_synth.workloads import CSA_PREFILL, layer_params
from gpu_helpers import DEV, act_tensor, assert_no_device_error, cache_view, check_scores, shape_of
from helpers import block_table

pytestmark = pytest.mark.gpu

W16 = dataclasses.replace(CSA_PREFILL, name="itk_bf16")
W8 = dataclasses.replace(CSA_PREFILL, key_fmt=C.CSLA_KEY_E4M3, name="itk_e4m3")


def _i32(x):
    return torch.as_tensor(np.asarray(x, np.int32), device=DEV)


def random_layer(w, lens, tag):
    """Slot i holds lens[i] tokens' worth of random index keys (bf16, or
    E4M3 codes with power-of-two scales) on a scattered page table."""
    bt, n_pages = block_table(w, lens, len(lens), seed_name=tag)
    lb = LayerBuffers(shape_of(w), len(lens), n_pages, bt.shape[1], DEV)
    lb.block_table.copy_(torch.from_numpy(bt))
    lb.len.copy_(_i32(lens))
    keys = TG.normal(w.seed, tag + "/keys", (n_pages, 32, w.dI), device=DEV)
    if w.key_fmt == C.CSLA_KEY_E4M3:
        lb.kidx.copy_((2.0 * keys).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8))
        ex = (TG.uniform(w.seed, tag + "/kexp", n_pages * 32, device=DEV) * 5).floor() - 8
        lb.kscale.copy_(torch.exp2(ex).to(torch.float32).reshape(n_pages, 32))
    else:
        lb.kidx.copy_(keys.to(torch.bfloat16).view(torch.int16))
    return lb


def inputs(w, B, tag, zero_weights=False):
    p = layer_params(w)
    cq = TG.normal(w.seed, tag + "/cq", (B, w.dc), device=DEV).to(torch.bfloat16)
    hw = TG.normal(w.seed, tag + "/hw", (B, w.HI), device=DEV).to(torch.float32)
    if zero_weights:
        hw.zero_()   # every score 0: all keys tie
    return cq, act_tensor(w, p["W_iq"]), hw


def two_calls(w, lb, slots, B, max_len, cq, W, hw, k, qs):
    stride = max_len // w.m
    scores = torch.full((B, stride), float("nan"), dtype=torch.float32, device=DEV)
    wsb = C.csla_workspace_size(lb.cfg(), C.CSLA_OP_INDEXER, B, max_len)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    C.csla_indexer_scores(lb.cfg(), lb.state(), lb.cache(), slots, B, max_len, cq, C.CSLA_BF16, W, C.CSLA_BF16, hw,
                          scores, stride, ws, wsb, qs=qs)
    idx = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    C.csla_topk_select(lb.cfg(), lb.state(), slots, B, max_len, scores, stride, k, idx, qs=qs)
    return idx, scores


def fused(w, lb, slots, B, max_len, cq, W, hw, k, qs):
    """idx of csla_indexer_topk and each row's fallback flag (read from the
    call's workspace: query terms, sample scores, thresholds, four counts per
    row, flags)."""
    stride = max_len // w.m
    scores = torch.full((B, stride), float("nan"), dtype=torch.float32, device=DEV)
    wsb = C.csla_workspace_size(lb.cfg(), C.CSLA_OP_INDEXER_TOPK, B, max_len)
    ws = torch.full((wsb,), 0xA5, dtype=torch.uint8, device=DEV)   # no zero-initialised scratch assumed
    idx = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    C.csla_indexer_topk(lb.cfg(), lb.state(), lb.cache(), slots, B, max_len, cq, C.CSLA_BF16, W, C.CSLA_BF16, hw,
                        k, idx, scores, stride, ws, wsb, qs=qs)
    off = C.indexer_topk_layout(B, w.HI, w.dI)["flags"]
    flags = ws[off:off + 4 * B].view(torch.int32).cpu().numpy()
    return idx, flags


def check(w, lb, slots, B, max_len, k, tag, qs=None, zero_weights=False, n_rows=None, oracle_rows=(),
          score_rows=()):
    """score_rows: rows whose stored scores (the two-call path's) are also
    checked against the oracle's index scores (one request in slot 0)."""
    cq, W, hw = inputs(w, B, tag, zero_weights)
    want, scores = two_calls(w, lb, slots, B, max_len, cq, W, hw, k, qs)
    got, flags = fused(w, lb, slots, B, max_len, cq, W, hw, k, qs)
    torch.cuda.synchronize()
    assert_no_device_error()
    g, e = got.cpu().numpy(), want.cpu().numpy()
    for b in range(B):
        assert np.array_equal(g[b], e[b]), (b, int(np.sum(g[b] != e[b])))
    for b in oracle_rows:
        n = int(n_rows[b])
        sc = scores[b, :n].cpu().numpy().astype(np.float64)
        assert np.array_equal(g[b], oracle.topk(sc, k)), b
    if score_rows:
        keys = cache_view(w, lb).gather_keys(0, int(max(n_rows[b] for b in score_rows)))
        cqh, Wh, hwh = (t.to(torch.float64).cpu().numpy() for t in (cq, W, hw))
        for b in score_rows:
            n = int(n_rows[b])
            qI = oracle.index_query(cqh[b], Wh, w.HI, w.dI)
            check_scores(scores[b, :n].cpu().numpy().astype(np.float64), oracle.index_scores(qI, hwh[b], keys[:n]))
    return flags


def test_long_query_rows_through_the_sample_threshold():
    """4096-token chunk rows after a 40000-token prefix scaled down to 23
    rows (groups of 5 with a ragged tail): ~10000 entries per row."""
    L0, T, k = 40000, 23, 1024
    lb = random_layer(W16, [L0 + T], "itk_a")
    q_len = np.arange(L0 + 1, L0 + T + 1)
    qs = C.queries(_i32(q_len), one_request=True)
    flags = check(W16, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_a", qs=qs, n_rows=q_len // 4,
                  oracle_rows=(0, T - 1))
    assert (flags == 0).sum() >= T - 1, flags   # the candidates sufficed (no stored scores)


def test_prefill_length_rows_top2048():
    """Rows of ~65500 entries (the 262144-token prefix), k = 2048."""
    L0, T, k = 262144 - 40, 11, 2048
    lb = random_layer(W16, [L0 + T], "itk_b")
    q_len = np.arange(L0 + 1, L0 + T + 1)
    flags = check(W16, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_b",
                  qs=C.queries(_i32(q_len), one_request=True), n_rows=q_len // 4, oracle_rows=(5,))
    assert (flags == 0).sum() >= T - 1, flags


def test_e4m3_keys_query_rows():
    L0, T, k = 80000, 9, 1024
    lb = random_layer(W8, [L0 + T], "itk_c")
    q_len = np.arange(L0 + 1, L0 + T + 1)
    check(W8, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_c", qs=C.queries(_i32(q_len), one_request=True),
          n_rows=q_len // 4, oracle_rows=(4,))


def test_decode_rows_of_several_requests():
    """One row per request: no entries, k < n <= 6144 (every entry a
    candidate), and long rows (sample threshold)."""
    lens = [3, 5000, 40000, 100000, 33000, 64004]
    lb = random_layer(W16, lens, "itk_d")
    B = len(lens)
    n_rows = [L // 4 for L in lens]
    check(W16, lb, torch.arange(B, dtype=torch.int32, device=DEV), B, max(lens), 512, "itk_d", n_rows=n_rows,
          oracle_rows=(1, 3))


@pytest.mark.parametrize("w", [W16, W8])
def test_ties_fall_back_or_break_by_entry(w):
    """Every score 0.  Rows of more than 6144 entries keep too many
    candidates and take the stored-score path (a few CTAs per row group,
    each walking a run of tiles); rows of fewer keep them all and break the
    tie by entry."""
    lens = [100000, 5000, 33000, 2100]
    lb = random_layer(w, lens, "itk_e")
    B = len(lens)
    flags = check(w, lb, torch.arange(B, dtype=torch.int32, device=DEV), B, max(lens), 512, "itk_e",
                  zero_weights=True, n_rows=[L // 4 for L in lens], oracle_rows=(0, 1))
    assert list(flags) == [1, 0, 1, 0], flags


def test_ties_on_query_rows_fall_back():
    L0, T, k = 60000, 7, 1024
    lb = random_layer(W16, [L0 + T], "itk_f")
    q_len = np.arange(L0 + 1, L0 + T + 1)
    flags = check(W16, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_f", qs=C.queries(_i32(q_len), one_request=True),
                  zero_weights=True, n_rows=q_len // 4, oracle_rows=(3,))
    assert list(flags) == [1] * T, flags


def test_full_size_prefill_chunk():
    """The bench's prefill chunk shape: 4096 query rows of one request after
    a 262144-token prefix (~66 K entries per row), k = 1024, in the launch
    configuration the bench times (5 rows per key tile, runs of tiles per
    CTA).  idx equal to the two calls' for every row; a few rows against
    the oracle's top-k of the stored scores."""
    L0, T, k = 262144, 4096, 1024
    lb = random_layer(W16, [L0 + T], "itk_full")
    q_len = np.arange(L0 + 1, L0 + T + 1)
    flags = check(W16, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_full",
                  qs=C.queries(_i32(q_len), one_request=True), n_rows=q_len // 4, oracle_rows=(0, 1777, T - 1))
    assert (flags == 0).sum() >= T - 8, int((flags != 0).sum())


@pytest.mark.parametrize("HI,dI,zero", [(4, 64, False), (8, 128, False), (4, 64, True)])
def test_query_rows_with_several_rows_per_epilogue_set(HI, dI, zero):
    """Fewer index heads: 16 (HI = 4) or 8 (HI = 8) query rows share a key
    tile and each epilogue warp set scores several of them, so the
    candidates take their places per (row, tile) from the row counters
    instead of a shared-memory stage; with zero head weights every row
    falls back to stored scores."""
    w = dataclasses.replace(W16, HI=HI, dI=dI, dc=256, name="itk_h%d" % HI)
    L0, T, k = 50000, 37, 512
    lb = random_layer(w, [L0 + T], "itk_g%d" % HI)
    q_len = np.arange(L0 + 1, L0 + T + 1)
    flags = check(w, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_g%d" % HI, qs=C.queries(_i32(q_len), one_request=True),
                  zero_weights=zero, n_rows=q_len // 4, oracle_rows=(0, T - 1), score_rows=(0, 17, T - 1))
    if zero:
        assert list(flags) == [1] * T, flags
    else:
        assert (flags == 0).sum() >= T - 1, flags


def test_fallback_through_the_streaming_top_k():
    """Rows longer than the cluster top-k holds (> 36864 entries) that fall
    back: the stored-score top-k is the streaming kernel, which skips the
    rows that were not flagged (the short row here)."""
    lens = [160000, 3000, 150001]
    lb = random_layer(W16, lens, "itk_s")
    B = len(lens)
    flags = check(W16, lb, torch.arange(B, dtype=torch.int32, device=DEV), B, max(lens), 1024, "itk_s",
                  zero_weights=True, n_rows=[L // 4 for L in lens], oracle_rows=(0, 2))
    assert list(flags) == [1, 0, 1], flags


def test_scores_rising_with_position():
    """Keys scaled up with their entry index, so that the top-k crowd into
    the last part of every row: the candidates come from a few tiles (the
    warps there stage and move out many of them), the sample still sees
    the whole row."""
    L0, T, k = 120000, 13, 1024
    lens = [L0 + T]
    lb = random_layer(W16, lens, "itk_p")
    bt = lb.block_table.cpu().numpy()[0]
    n = (L0 + T) // 4
    scale = torch.ones((lb.n_pages, 32), dtype=torch.float64)
    for c, pg in enumerate(bt):
        if pg >= 0:
            e = 32 * c + torch.arange(32, dtype=torch.float64)
            scale[int(pg)] = 1.0 + 3.0 * (e / n) ** 4
    keys = lb.kidx.view(torch.bfloat16).to(torch.float64) * scale.to(DEV)[:, :, None]
    lb.kidx.copy_(keys.to(torch.bfloat16).view(torch.int16))
    q_len = np.arange(L0 + 1, L0 + T + 1)
    flags = check(W16, lb, _i32(np.zeros(T)), T, L0 + T, k, "itk_p", qs=C.queries(_i32(q_len), one_request=True),
                  n_rows=q_len // 4, oracle_rows=(0, T - 1))
    assert (flags == 0).sum() >= T - 1, flags
