"""csla_csa_decode_step (the append overlapped with the indexer's scoring of
the entries that were already complete) against the four separate calls:
identical caches, scores, top-k lists and outputs, bit for bit, over decode
steps that close blocks and steps that do not."""
import dataclasses

import numpy as np
import pytest
import torch

from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import CompressParams
from csla_synth.workloads import CSA_DECODE, CSA_TINY, layer_params, step_inputs, token_stream
from gpu_helpers import DEV, act_tensor, assert_no_device_error, upload_layer
from helpers import oracle_cache

pytestmark = pytest.mark.gpu


def _f32(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32, device=DEV)


class Layer:
    def __init__(self, w, lens, max_len):
        cv, p = oracle_cache(w, lens)
        self.lb = upload_layer(w, cv, lens)
        self.cp = CompressParams(p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"), p.get("gbi"), DEV)
        self.p = p
        B = len(lens)
        cfg = self.lb.cfg()
        self.stride = max_len // w.m
        self.scores = torch.full((B, self.stride), float("nan"), dtype=torch.float32, device=DEV)
        self.idx = torch.full((B, w.k), -7, dtype=torch.int32, device=DEV)
        self.out = torch.full((B, w.H, w.D), float("nan"), dtype=torch.float32, device=DEV)
        self.wsi_b = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, max_len)
        self.wsi = torch.zeros(self.wsi_b, dtype=torch.uint8, device=DEV)
        self.wsa_b = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, B, w.k)
        self.wsa = torch.zeros(self.wsa_b, dtype=torch.uint8, device=DEV)
        self.wss_b = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_DECODE_STEP, B, w.k)
        self.wss = torch.zeros(self.wss_b, dtype=torch.uint8, device=DEV)


def _state(L):
    h = L.lb.host_view()
    return {k: np.array(v) for k, v in h.items()}


@pytest.mark.parametrize("w,lens", [
    (dataclasses.replace(CSA_TINY, B=3, L=700, name="step_tiny"), [700, 301, 6]),
    (dataclasses.replace(CSA_DECODE, B=4, L=3000, name="step_big"), [2999, 1998, 513, 3]),
])
def test_decode_step_equals_separate_calls(w, lens):
    B = len(lens)
    n_steps = 6
    max_len = max(lens) + n_steps
    A, F = Layer(w, lens, max_len), Layer(w, lens, max_len)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    dt = C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32
    W = act_tensor(w, A.p["W_iq"])
    sink, gq = _f32(A.p["sink"]), _f32(A.p["gamma_q"])
    for step in range(n_steps):
        si = step_inputs(w, 40 + step)
        kv = act_tensor(w, np.stack([token_stream(w, b, L + step, L + step + 1)["kv"] for b, L in enumerate(lens)]))
        ki = act_tensor(w, np.stack([token_stream(w, b, L + step, L + step + 1)["idx"] for b, L in enumerate(lens)]))
        cq, q = act_tensor(w, si["cq"][:B]), act_tensor(w, si["q"][:B])
        hw = _f32(si["head_w"][:B])
        cfg = A.lb.cfg()
        C.csla_compress_append(cfg, A.lb.state(), A.lb.cache(), slots, B, 1, kv, ki, dt, A.cp.struct())
        C.csla_indexer_scores(cfg, A.lb.state(), A.lb.cache(), slots, B, max_len, cq, dt, W, dt, hw, A.scores,
                              A.stride, A.wsi, A.wsi_b)
        C.csla_topk_select(cfg, A.lb.state(), slots, B, max_len, A.scores, A.stride, w.k, A.idx)
        C.csla_csa_attend(cfg, A.lb.state(), A.lb.cache(), slots, B, q, dt, A.idx, w.k, sink, gq, A.out,
                          C.CSLA_F32, C.CSLA_VARIANT_AUTO, A.wsa, A.wsa_b)
        C.csla_csa_decode_step(F.lb.cfg(), F.lb.state(), F.lb.cache(), slots, B, 1, max_len, kv, ki, dt,
                               F.cp.struct(), cq, dt, W, dt, hw, F.scores, F.stride, w.k, F.idx, q, dt,
                               sink, gq, F.out, C.CSLA_F32, C.CSLA_VARIANT_AUTO, F.wsi, F.wsi_b, F.wss, F.wss_b)
        assert_no_device_error()
        sa, sf = _state(A), _state(F)
        for k in sa:
            assert np.array_equal(sa[k], sf[k]), (step, k)
        for b, L in enumerate(lens):
            nv = (L + step + 1) // w.m
            assert torch.equal(A.scores[b, :nv], F.scores[b, :nv]), (step, b)
        assert torch.equal(A.idx, F.idx), step
        assert bool(torch.isfinite(A.out).all()), step
        assert torch.equal(A.out.view(torch.int32), F.out.view(torch.int32)), step
