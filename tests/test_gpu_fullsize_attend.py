"""Attention parity at the full set sizes of the HCA decode and CSA prefill
workloads, where the canonical chunking takes its larger branches:

  * HCA decode, 4 requests at 2^20 tokens (8192 compressed entries + 128
    window rows = 8320 rows per request, lengths staggered 16 tokens apart
    as in the benchmark): both kernel variants, every request, against the
    oracle's fp64 attention over the same decoded rows.
  * CSA query rows of one request at top-k 1024 (1152-row sets, the prefill
    chunk's configuration) and top-k 2048 (the largest supported k), with
    per-row visible lengths and window rows read from a chunk buffer
    (csla_queries), both variants.

Pages: 硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力 (HCA: every entry
plus the window; CSA: top-k 512/1024 plus the window; sink, RoPE on the last
64 dims, bf16/fp8 cache).

Caches hold quantised rows of N(0,1) content through RMSNorm and RoPE at
their positions (the compressor's output distribution), written on the host
by the oracle and uploaded, so both sides decode the same bytes; the
compressor itself is covered by the compress parity tests."""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import LayerBuffers, LayerShape
from csla_synth import normal, permutation
from gpu_helpers import DEV, assert_no_device_error, check_out

pytestmark = pytest.mark.gpu

D, H, DR = 512, 64, 64
RB = oracle.row_bytes(D, DR)


def _rows(seed, name, positions, gamma):
    """Quantised rows (and scales) of N(0,1) vectors through RMSNorm*gamma
    and RoPE at the given positions."""
    x = normal(seed, name, (len(positions), D))
    rows = np.zeros((len(positions), RB), np.uint8)
    sc = np.zeros(len(positions), np.float32)
    for i, p in enumerate(positions):
        rows[i], sc[i] = oracle.window_row(x[i], gamma, int(p))
    return rows, sc


def _params(seed):
    gamma = (1.0 + 0.1 * normal(seed, "fs/gamma_kv", (D,))).astype(np.float32).astype(np.float64)
    gamma_q = (1.0 + 0.1 * normal(seed, "fs/gamma_q", (D,))).astype(np.float32).astype(np.float64)
    sink = normal(seed, "fs/sink", (H,)).astype(np.float32).astype(np.float64)
    return gamma, gamma_q, sink


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float64).to(torch.bfloat16)


def _filled(m, lens, seed):
    """Oracle cache view (and device copy) of len(lens) requests: every
    visible entry filled, the ring holding each request's last 128 tokens;
    physical pages a seeded permutation."""
    epp = 128 // m
    gamma, _, _ = _params(seed)
    need = [-(-L // 128) for L in lens]
    stride = max(need)
    n_pages = sum(need)
    perm = permutation(seed, "fs/pages", n_pages).astype(np.int32)
    bt = -np.ones((len(lens), stride), np.int32)
    rows = np.zeros((n_pages, epp, RB), np.uint8)
    scales = np.zeros((n_pages, epp), np.float32)
    win = np.zeros((len(lens), 128, RB), np.uint8)
    wsc = np.zeros((len(lens), 128), np.float32)
    k = 0
    for s, L in enumerate(lens):
        bt[s, :need[s]] = perm[k:k + need[s]]
        k += need[s]
        nv = L // m
        r, sc = _rows(seed, "fs/rows/%d" % s, np.arange(nv) * m, gamma)
        e = np.arange(nv)
        rows[bt[s, e // epp], e % epp] = r
        scales[bt[s, e // epp], e % epp] = sc
        pos = np.arange(max(0, L - 128), L)
        r, sc = _rows(seed, "fs/win/%d" % s, pos, gamma)
        win[s, pos % 128], wsc[s, pos % 128] = r, sc
    cv = oracle.CacheView(m, D, rows, scales, bt, win, wsc)
    shape = LayerShape(m=m, D=D, H=H, HI=16, dI=128, dc=1024)
    lb = LayerBuffers(shape, len(lens), n_pages, stride, DEV)
    lb.rows.copy_(torch.from_numpy(rows))
    lb.scales.copy_(torch.from_numpy(scales))
    lb.block_table.copy_(torch.from_numpy(bt))
    lb.win_rows.copy_(torch.from_numpy(win))
    lb.win_scales.copy_(torch.from_numpy(wsc))
    lb.len.copy_(torch.tensor(lens, dtype=torch.int32))
    torch.cuda.synchronize()
    return cv, lb


def _dev(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32, device=DEV)


def test_hca_full_size_matches_oracle():
    """4 x 2^20 tokens, m' = 128: 8320 / 8319 rows per request (26 chunks of
    320 rows), saturated and starved variants bit-identical, every request
    within the attention tolerance of the oracle."""
    seed, L = 2, 1 << 20
    lens = [L - 16 * b for b in range(4)]
    cv, lb = _filled(128, lens, seed)
    _, gamma_q, sink = _params(seed)
    q = _bf16(normal(seed, "fs/q", (len(lens), H, D)))
    qd = q.to(DEV)
    cfg = lb.cfg()
    ml = max(lens)
    wsb = C.csla_workspace_size(cfg, C.CSLA_OP_HCA_ATTEND, len(lens), ml)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    outs = {}
    for v in (C.CSLA_VARIANT_SATURATED, C.CSLA_VARIANT_STARVED, C.CSLA_VARIANT_AUTO):
        out = torch.full((len(lens), H, D), float("nan"), dtype=torch.float32, device=DEV)
        C.csla_hca_attend(cfg, lb.state(), lb.cache(), torch.arange(len(lens), dtype=torch.int32, device=DEV),
                          len(lens), ml, qd, C.CSLA_BF16, _dev(sink), _dev(gamma_q), out, C.CSLA_F32, v, ws, wsb)
        outs[v] = out
    torch.cuda.synchronize()
    assert_no_device_error()
    assert torch.equal(outs[1], outs[2]) and torch.equal(outs[1], outs[0]), "variants differ"
    got = outs[1].cpu().numpy().astype(np.float64)
    qn = q.double().numpy()
    for s, Ls in enumerate(lens):
        rows = cv.gather_set(s, Ls)
        assert rows.shape[0] == Ls // 128 + 128
        ref, _ = oracle.attend(qn[s], gamma_q, Ls - 1, rows, sink)
        check_out(got[s], ref)


@pytest.mark.parametrize("k", [1024, 2048])
def test_csa_query_rows_full_topk_match_oracle(k):
    """Query rows of one request with per-row visible lengths, top-k lists of
    k entries (seeded subsets of each row's visible entries) and window rows
    from a buffer indexed by position: k + 128 rows per set (320-row
    chunks), both variants bit-identical, every row against the oracle."""
    seed = 4
    L1 = 4 * k + 3000
    cv, lb = _filled(4, [L1], seed)
    gamma, gamma_q, sink = _params(seed)
    # window rows of every position 0..L1-1, by position (win_base = 0)
    buf, bsc = _rows(seed, "fs/buf", np.arange(L1), gamma)
    q_len = np.array([4 * k, 4 * k + 1, 4 * k + 517, L1 - 300, L1 - 1, L1], np.int32)
    T = len(q_len)
    idx = np.zeros((T, k), np.int32)
    for i, Lq in enumerate(q_len):
        nv = Lq // 4
        idx[i] = np.sort(permutation(seed, "fs/sel/%d" % i, nv)[:k])
    q = _bf16(normal(seed, "fs/pq", (T, H, D)))
    cfg = lb.cfg()
    qs = C.queries(torch.from_numpy(q_len).to(DEV), torch.from_numpy(buf).to(DEV), torch.from_numpy(bsc).to(DEV),
                   torch.zeros(T, dtype=torch.int32, device=DEV), L1)
    slots = torch.zeros(T, dtype=torch.int32, device=DEV)
    wsb = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, T, k)
    ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
    idx_d = torch.from_numpy(idx).to(DEV)
    outs = {}
    for v in (C.CSLA_VARIANT_SATURATED, C.CSLA_VARIANT_STARVED):
        out = torch.full((T, H, D), float("nan"), dtype=torch.float32, device=DEV)
        C.csla_csa_attend(cfg, lb.state(), lb.cache(), slots, T, q.to(DEV), C.CSLA_BF16, idx_d, k, _dev(sink),
                          _dev(gamma_q), out, C.CSLA_F32, v, ws, wsb, qs=qs)
        outs[v] = out
    torch.cuda.synchronize()
    assert_no_device_error()
    assert torch.equal(outs[1], outs[2]), "variants differ"
    got = outs[1].cpu().numpy().astype(np.float64)
    qn = q.double().numpy()
    for i, Lq in enumerate(q_len):
        sel = cv.gather_set(0, int(Lq), idx[i])[:k]          # the selected entries ...
        w0 = max(0, int(Lq) - 128)
        win = oracle.dequantize_rows(buf[w0:Lq], bsc[w0:Lq], D)   # ... then the window from the buffer
        rows = np.concatenate([sel, win])
        assert rows.shape[0] == k + 128
        ref, _ = oracle.attend(qn[i], gamma_q, int(Lq) - 1, rows, sink)
        check_out(got[i], ref)
