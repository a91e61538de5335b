"""GPU parity: csla_csa_attend / csla_hca_attend against the oracle's fp64
MQA with sink on the same decoded cache rows; exact widening of every E4M3
code; saturated and starved variants bit-identical; batch invariance."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import LayerBuffers, LayerShape
from csla_synth.workloads import CSA_DECODE, CSA_TINY, HCA_DECODE, layer_params, step_inputs
from gpu_helpers import DEV, act_tensor, assert_no_device_error, check_out, upload_layer
from helpers import oracle_cache

pytestmark = pytest.mark.gpu



def attend(w, lb, q, sink, gamma_q, lens, idx=None, variant=C.CSLA_VARIANT_AUTO, slots=None,
           out_dtype=torch.float32):
    B = q.shape[0]
    cfg = lb.cfg()
    slots = torch.arange(B, dtype=torch.int32, device=DEV) if slots is None else slots
    out = torch.full((B, w.H, w.D), float("nan"), dtype=out_dtype, device=DEV)
    odt = C.CSLA_F32 if out_dtype == torch.float32 else C.CSLA_BF16
    qdt = C.CSLA_BF16 if q.dtype == torch.bfloat16 else C.CSLA_F32
    if idx is not None:
        k = idx.shape[1]
        wsb = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, B, k)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=DEV)
        C.csla_csa_attend(cfg, lb.state(), lb.cache(), slots, B, q, qdt, idx, k, sink, gamma_q, out, odt,
                          variant, ws, wsb)
    else:
        ml = max(lens)
        wsb = C.csla_workspace_size(cfg, C.CSLA_OP_HCA_ATTEND, B, ml)
        ws = torch.zeros(max(wsb, 16), dtype=torch.uint8, device=DEV)
        C.csla_hca_attend(cfg, lb.state(), lb.cache(), slots, B, ml, q, qdt, sink, gamma_q, out, odt, variant,
                          ws, wsb)
    return out


def _dev(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32, device=DEV)


def test_every_e4m3_code_widens_exactly():
    """Window of one token whose fp8 dims hold every finite E4M3 code with
    scale 1 and whose RoPE dims hold values the f16 operand carries exactly
    at that scale: with the sink at -1e30 the output is that row, exactly."""
    shape = LayerShape(m=128, D=512, H=8)
    lb = LayerBuffers(shape, 1, 1, 1, DEV)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    row = np.zeros(576, np.uint8)
    row[:448] = np.resize(codes, 448)
    # 1, -1, 2^-10, 2992: each / 256 is an f16 value
    rope = np.array([0x3F80, 0xBF80, 0x3A80, 0x453B] * 16, np.uint16)
    row[448:] = rope.view(np.uint8)
    lb.win_rows[0, 0] = torch.from_numpy(row).to(DEV)
    lb.win_scales[0, 0] = 1.0
    lb.len[0] = 1
    q = torch.zeros((1, 8, 512), dtype=torch.float32, device=DEV)
    q[..., 0] = 1.0
    out = attend(dataclasses.replace(HCA_DECODE, H=8), lb, q, _dev(np.full(8, -1e30)),
                 _dev(np.ones(512)), [1])
    assert_no_device_error()
    want = oracle.dequantize(row, 1.0, 512)
    assert want[449] == -1.0 and want[450] == 2.0 ** -10 and want[451] == 2992.0
    got = out.cpu().numpy().astype(np.float64)[0]
    for h in range(8):
        assert np.array_equal(got[h], want), np.nonzero(got[h] != want)


def test_row_outside_operand_range_is_masked_and_flagged():
    """A window row whose fp8 scale is beyond the operand range (|x| up to
    448 * 100) is masked and sets CSLA_DEVERR_RANGE; the output is the
    attention over the remaining rows, finite."""
    w = dataclasses.replace(HCA_DECODE, H=8, B=1, L=3, name="range")
    shape = LayerShape(m=128, D=512, H=8)
    lb = LayerBuffers(shape, 1, 1, 1, DEV)
    rng = np.random.default_rng(5)
    rows = rng.integers(0, 0x7E, size=(3, 576)).astype(np.uint8)
    rows[:, 448:] = 0
    scales = np.array([0.01, 100.0, 0.02], np.float32)
    lb.win_rows[0, :3] = torch.from_numpy(rows).to(DEV)
    lb.win_scales[0, :3] = torch.from_numpy(scales).to(DEV)
    lb.len[0] = 3
    q = torch.zeros((1, 8, 512), dtype=torch.float32, device=DEV)
    q[..., :8] = 1.0
    sink = np.zeros(8)
    out = attend(w, lb, q, _dev(sink), _dev(np.ones(512)), [3])
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_ERR_DEVICE and bits == C.CSLA_DEVERR_RANGE, (rc, bits)
    kept = np.stack([oracle.dequantize(rows[i], scales[i], 512) for i in (0, 2)])
    ref, _ = oracle.attend(q.cpu().numpy()[0].astype(np.float64), np.ones(512), 2, kept, sink)
    got = out.cpu().numpy().astype(np.float64)[0]
    assert np.all(np.isfinite(got))
    check_out(got, ref)


CSA_SMALL = dataclasses.replace(CSA_TINY, B=3, L=2048, name="att_csa_tiny")
CSA_BIG = dataclasses.replace(CSA_DECODE, B=2, L=6000, name="att_csa_big")
HCA_SMALL = dataclasses.replace(HCA_DECODE, B=4, L=40000, name="att_hca")


def _oracle_idx(w, cv, s, L, si, p):
    nv = L // w.m
    qI = oracle.index_query(si["cq"][s], p["W_iq"], w.HI, w.dI)
    return oracle.topk(oracle.index_scores(qI, si["head_w"][s], cv.gather_keys(s, nv)), w.k)


@pytest.mark.parametrize("w,lens", [
    (CSA_SMALL, [2048, 300, 5]),
    (CSA_BIG, [6000, 130]),
    (dataclasses.replace(CSA_SMALL, H=5, name="att_csa_h5"), [2048, 77]),   # odd head count
])
def test_csa_attend_matches_oracle(w, lens):
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 5)
    idx_np = np.stack([_oracle_idx(w, cv, s, L, si, p) for s, L in enumerate(lens)])
    idx = torch.as_tensor(idx_np, dtype=torch.int32, device=DEV)
    q = act_tensor(w, si["q"][:len(lens)])
    outs = {}
    for v in (C.CSLA_VARIANT_SATURATED, C.CSLA_VARIANT_STARVED):
        outs[v] = attend(w, lb, q, _dev(p["sink"]), _dev(p["gamma_q"]), lens, idx=idx, variant=v)
    assert_no_device_error()
    assert torch.equal(outs[1], outs[2]), "variants differ"
    got = outs[1].cpu().numpy().astype(np.float64)
    for s, L in enumerate(lens):
        rows = cv.gather_set(s, L, idx_np[s])
        ref, _ = oracle.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"], w.eps, w.theta, w.d_rope)
        check_out(got[s], ref)


@pytest.mark.parametrize("lens", [[40000, 129, 1, 17000], [128, 255, 256, 8320]])
def test_hca_attend_matches_oracle(lens):
    w = dataclasses.replace(HCA_SMALL, B=len(lens))
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 6)
    q = act_tensor(w, si["q"])
    outs = {}
    for v in (C.CSLA_VARIANT_SATURATED, C.CSLA_VARIANT_STARVED):
        outs[v] = attend(w, lb, q, _dev(p["sink"]), _dev(p["gamma_q"]), lens, variant=v)
    assert_no_device_error()
    assert torch.equal(outs[1], outs[2]), "variants differ"
    got = outs[1].cpu().numpy().astype(np.float64)
    for s, L in enumerate(lens):
        rows = cv.gather_set(s, L)
        ref, _ = oracle.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"], w.eps, w.theta, w.d_rope)
        check_out(got[s], ref)


def test_hca_batch_invariance():
    """A request's output is bit-identical alone, in a batch, at any batch
    position, and under either variant."""
    lens = [20000, 300, 9000, 129]
    w = dataclasses.replace(HCA_SMALL, B=len(lens))
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    si = step_inputs(w, 7)
    q = act_tensor(w, si["q"])
    sink, g = _dev(p["sink"]), _dev(p["gamma_q"])
    full = attend(w, lb, q, sink, g, lens, variant=C.CSLA_VARIANT_STARVED)
    for s in range(len(lens)):
        alone = attend(w, lb, q[s:s + 1].contiguous(), sink, g, lens,
                       slots=torch.tensor([s], dtype=torch.int32, device=DEV), variant=C.CSLA_VARIANT_SATURATED)
        assert torch.equal(alone[0], full[s]), s
    perm = [2, 0, 3, 1]
    shuffled = attend(w, lb, q[perm].contiguous(), sink, g, lens,
                      slots=torch.tensor(perm, dtype=torch.int32, device=DEV))
    for i, s in enumerate(perm):
        assert torch.equal(shuffled[i], full[s])
    assert_no_device_error()
