"""Batch-invariance stress (the contract's invariance workload): 64 ragged
decode requests with contexts log-uniform in [1K, 1M] tokens, a CSA layer
(m=4, top-k 512, indexer) and an HCA layer (m'=128), head_dim 512, 64 heads.
Every request is decoded alone and inside 8 shuffled batchings, with both
attention variants; its top-k indices and outputs must be identical bit for
bit in every run (QbitAI article on batch invariance: a token's result must
not depend on the batch it is served in).

Caches are filled directly with valid random rows (random E4M3 codes, the two
NaN codes excluded, N(0,1) bf16 RoPE dims and index keys, scales in [0.005,
0.015]): invariance does not depend on how the rows were produced, and the
compressor itself has no cross-request arithmetic (one CTA per token or
block of one request)."""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import LayerBuffers, LayerShape
from csla_synth import uniform
from gpu_helpers import DEV, assert_no_device_error

pytestmark = pytest.mark.gpu

N_REQ, H, D, K = 64, 64, 512, 512
SEED = 5


def _lengths():
    u = uniform(SEED, "invariance/len", (N_REQ,))
    return [int(math.exp(math.log(1024) + x * math.log(1024))) for x in u]


def _fill_layer(shape, lens, gen):
    """A layer whose caches hold valid random rows for every visible entry
    and window slot of every request (slot r = request r)."""
    pages = [-(-L // 128) for L in lens]
    bt_stride, n_pages = max(pages), sum(pages)
    lb = LayerBuffers(shape, len(lens), n_pages, bt_stride, DEV)
    perm = torch.randperm(n_pages, generator=gen, device=DEV).to(torch.int32)
    bt = torch.full((len(lens), bt_stride), -1, dtype=torch.int32, device=DEV)
    k = 0
    for r, n in enumerate(pages):
        bt[r, :n] = perm[k:k + n]
        k += n
    lb.block_table.copy_(bt)
    dn = D - 64

    def fill_rows(dst):
        # random bytes for the fp8 dims (the two NaN codes moved to their
        # neighbours), N(0,1) bf16 for the RoPE dims; in slices of 64K rows
        for a in range(0, dst.shape[0], 1 << 16):
            part = dst[a:a + (1 << 16)]
            c = torch.randint(0, 256, (part.shape[0], dn), generator=gen, device=DEV, dtype=torch.uint8)
            c[c == 0x7F] = 0x7E
            c[c == 0xFF] = 0xFE
            part[:, :dn] = c
            part[:, dn:] = torch.randn((part.shape[0], 64), generator=gen, device=DEV).to(torch.bfloat16).view(
                torch.uint8)

    fill_rows(lb.rows.view(-1, dn + 128))
    lb.scales.copy_(0.005 + 0.01 * torch.rand(lb.scales.shape, generator=gen, device=DEV))
    if shape.m == 4:
        lb.kidx.copy_(torch.randn(lb.kidx.shape, generator=gen, device=DEV).to(torch.bfloat16).view(torch.int16))
    fill_rows(lb.win_rows.view(-1, dn + 128))
    lb.win_scales.copy_(0.005 + 0.01 * torch.rand(lb.win_scales.shape, generator=gen, device=DEV))
    lb.len.copy_(torch.tensor(lens, dtype=torch.int32))
    torch.cuda.synchronize()
    return lb


def _batchings(n_ways):
    """n_ways shuffled partitions of the requests into ragged batches."""
    rng = np.random.default_rng(SEED)
    out = []
    for _ in range(n_ways):
        order = rng.permutation(N_REQ)
        cuts, i = [], 0
        while i < N_REQ:
            s = int(rng.integers(1, 33))
            cuts.append([int(x) for x in order[i:i + s]])
            i += s
        out.append(cuts)
    return out


def test_invariance_stress_csa_and_hca():
    gen = torch.Generator(device=DEV)
    gen.manual_seed(SEED)
    lens = _lengths()
    max_len = max(lens)
    csa = _fill_layer(LayerShape(m=4, D=D, H=H, HI=16, dI=128, dc=1024), lens, gen)
    hca = _fill_layer(LayerShape(m=128, D=D, H=H), lens, gen)
    q = torch.randn((N_REQ, H, D), generator=gen, device=DEV).to(torch.bfloat16)
    cq = torch.randn((N_REQ, 1024), generator=gen, device=DEV).to(torch.bfloat16)
    head_w = torch.randn((N_REQ, 16), generator=gen, device=DEV)
    W_iq = (torch.randn((16 * 128, 1024), generator=gen, device=DEV) / 32).to(torch.bfloat16)
    sink = torch.randn((H,), generator=gen, device=DEV)
    gamma_q = 1.0 + 0.1 * torch.randn((D,), generator=gen, device=DEV)
    stride = max_len // 4

    def run(ids, variant):
        B = len(ids)
        slots = torch.tensor(ids, dtype=torch.int32, device=DEV)
        sel = slots.long()
        cfg = csa.cfg()
        wsi = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, max_len)
        ws_i = torch.zeros(max(wsi, 16), dtype=torch.uint8, device=DEV)
        scores = torch.zeros((B, stride), dtype=torch.float32, device=DEV)
        C.csla_indexer_scores(cfg, csa.state(), csa.cache(), slots, B, max_len, cq[sel].contiguous(),
                              C.CSLA_BF16, W_iq, C.CSLA_BF16, head_w[sel].contiguous(), scores, stride, ws_i, wsi)
        idx = torch.full((B, K), -7, dtype=torch.int32, device=DEV)
        C.csla_topk_select(cfg, csa.state(), slots, B, max_len, scores, stride, K, idx)
        wsa = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, B, K)
        ws_a = torch.zeros(max(wsa, 16), dtype=torch.uint8, device=DEV)
        out_c = torch.empty((B, H, D), dtype=torch.bfloat16, device=DEV)
        qb = q[sel].contiguous()
        C.csla_csa_attend(cfg, csa.state(), csa.cache(), slots, B, qb, C.CSLA_BF16, idx, K, sink, gamma_q,
                          out_c, C.CSLA_BF16, variant, ws_a, wsa)
        hcfg = hca.cfg()
        wsh = C.csla_workspace_size(hcfg, C.CSLA_OP_HCA_ATTEND, B, max_len)
        ws_h = torch.zeros(max(wsh, 16), dtype=torch.uint8, device=DEV)
        out_h = torch.empty((B, H, D), dtype=torch.bfloat16, device=DEV)
        C.csla_hca_attend(hcfg, hca.state(), hca.cache(), slots, B, max_len, qb, C.CSLA_BF16, sink, gamma_q,
                          out_h, C.CSLA_BF16, variant, ws_h, wsh)
        return idx, out_c, out_h

    variants = (C.CSLA_VARIANT_SATURATED, C.CSLA_VARIANT_STARVED)
    ref = {}
    for r in range(N_REQ):                      # alone, reference variant
        ref[r] = run([r], variants[0])
    torch.cuda.synchronize()
    assert_no_device_error()
    for r in range(N_REQ):                      # top-k sets are complete and ascending
        i = ref[r][0][0]
        nv = lens[r] // 4
        assert int((i >= 0).sum()) == min(K, nv)
        v = i[i >= 0]
        assert bool((v[1:] > v[:-1]).all()) and int(v[-1]) < nv
    runs = [([[r] for r in range(N_REQ)], variants[1])]
    runs += [(b, v) for b in _batchings(8) for v in variants]
    for batches, variant in runs:
        for ids in batches:
            idx, oc, oh = run(ids, variant)
            for j, r in enumerate(ids):
                assert torch.equal(idx[j], ref[r][0][0]), ("csa idx", r, variant)
                assert torch.equal(oc[j], ref[r][1][0]), ("csa out", r, variant)
                assert torch.equal(oh[j], ref[r][2][0]), ("hca out", r, variant)
    assert_no_device_error()
