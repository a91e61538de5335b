"""Parity at the full CSA decode workload, in bench.py's launch
configuration: 8 requests x 131072 tokens (m=4: 32768 entries each), 64
heads, D=512, 16 index heads of 128, dc=1024, top-k 512, window 128.  The
layer is built and one decode step is run exactly as bench.py does (caches
appended by csla_compress_append from the device token streams, the four
calls on the whole batch, automatic (starved) attention).  The oracle then
recomputes, for a sampled request, from the same seeded streams evaluated
on the CPU: its newest window row, newest compressed entry and index key,
all 32768 index scores, its top-k set and its attention output."""
import math

import numpy as np
import pytest
import torch

import bench
import oracle
from csla_synth import normal, torch_gen
from gpu_helpers import DEV, assert_bf16_close, assert_no_device_error, compare_rows

pytestmark = pytest.mark.gpu

SEED = 1
SAMPLE = 4            # a request whose append closes a block, at the full context
REL_TOL, GAP_TOL, MAX_ABS = 1e-3, 1e-4, 1e-2


def _f32(x):
    return np.asarray(x, np.float32).astype(np.float64)


def _bf16(t):
    return t.to(torch.bfloat16).double().numpy()


def test_csa_decode_full_size_sampled():
    kw = dict(bench.CSA)
    B, L, D, dI, m, H, k = kw["B"], kw["L"], kw["D"], kw["dI"], kw["m"], kw["H"], kw["k"]
    L0s = [L - 1 - (b % m) for b in range(B)]
    dev = torch.device(DEV)
    lb, cp, params = bench.build_layer(kw, B, L0s, SEED, 0, dev)
    inputs = bench.step_inputs(kw, B, 1, SEED, 0, dev)
    st = bench.CsaStep(lb, cp, params, kw, 0, dev)
    for call in st.calls:
        call(inputs[0])
    torch.cuda.synchronize()
    assert_no_device_error()

    s = SAMPLE
    L0 = L0s[s]
    Ls = L0 + 1                      # context after this step's append
    nv = Ls // m
    assert Ls % m == 0               # the sampled request closes a block this step
    # the layer parameters exactly as bench.build_layer makes them (fp32 arithmetic)
    g32 = lambda name, shp, std=1.0: np.asarray(normal(SEED, name, shp, std=std), np.float32)
    gam = lambda name: (np.float32(1.0) + np.float32(0.1) * g32(name, (D,))).astype(np.float64)
    gamma_kv, gamma_q = gam("gamma_kv"), gam("gamma_q")
    wg, gb = _f32(g32("wg", (D,), 1.0 / D ** 0.5)), _f32(g32("gb", (m,)))
    wgi, gbi = _f32(g32("wgi", (dI,), 1.0 / dI ** 0.5)), _f32(g32("gbi", (m,)))
    sink = _f32(g32("sink", (H,)))
    # the request's raw streams, positions 0..L0-1, then this step's token
    kv = np.concatenate([_bf16(torch_gen.normal(SEED, "kv/0/%d" % s, (L0, D), device="cpu")),
                         _bf16(torch_gen.normal(SEED, "kvn/0/0", (B, 1, D), device="cpu"))[s]])
    ki = np.concatenate([_bf16(torch_gen.normal(SEED, "idx/0/%d" % s, (L0, dI), device="cpu")),
                         _bf16(torch_gen.normal(SEED, "kin/0/0", (B, 1, dI), device="cpu"))[s]])
    q = _bf16(torch_gen.normal(SEED, "q/0/0", (B, H, D), device="cpu"))[s]
    cq = _bf16(torch_gen.normal(SEED, "cq/0/0", (B, kw["dc"]), device="cpu"))[s]
    hw = _f32(torch_gen.normal(SEED, "hw/0/0", (B, kw["HI"]), device="cpu").numpy())[s]
    W = _bf16(torch_gen.normal(SEED, "W_iq", (kw["HI"] * dI, kw["dc"]), device="cpu", std=1.0 / kw["dc"] ** 0.5))

    h = lb.host_view()
    bt = h["block_table"][s]
    epp = 128 // m
    # newest window row and newest compressed entry + index key
    y = oracle.rope(oracle.rmsnorm(kv[Ls - 1], gamma_kv, 1e-6), Ls - 1, 10000.0, 64)
    compare_rows(h["win_rows"][s, (Ls - 1) % 128], h["win_scales"][s, (Ls - 1) % 128], y, D)
    b = nv - 1
    c, _ = oracle.gate_pool(kv[b * m:(b + 1) * m], wg, gb)
    y = oracle.rope(oracle.rmsnorm(c, gamma_kv, 1e-6), b * m, 10000.0, 64)
    pg = bt[b // epp]
    compare_rows(h["rows"][pg, b % epp], h["scales"][pg, b % epp], y, D)
    xi = ki[b * m:(b + 1) * m]
    assert_bf16_close(h["kidx"][pg, b % epp], oracle.index_key(xi, wgi, gbi), 1e-5 * float(np.max(np.abs(xi))))

    # every index key of the request, then every index score.  The GPU's keys
    # (fp32 pooling, one bf16 rounding) may differ from the oracle's by one
    # bf16 ulp per dim, so a score may move by up to
    #   bound_s = 2^-7 * sum_j |w_j| sum_e |q_je k_se|   (ReLU is 1-Lipschitz)
    # on top of the indexer's own 1e-3 relative error.
    kbits = np.stack([oracle.index_key(ki[e * m:(e + 1) * m], wgi, gbi) for e in range(nv)])
    gk = h["kidx"][bt[np.arange(nv) // epp], np.arange(nv) % epp]
    for e0 in range(0, nv, 4096):
        xmax = float(np.max(np.abs(ki[e0 * m:(e0 + 4096) * m])))
        assert_bf16_close(gk[e0:e0 + 4096].reshape(-1), kbits[e0:e0 + 4096].reshape(-1), 1e-5 * xmax)
    keys = (kbits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    qI = oracle.index_query(cq, W, kw["HI"], dI).reshape(kw["HI"], dI)
    ref = oracle.index_scores(qI, hw, keys)
    bound = 2.0 ** -7 * (np.abs(keys) @ np.abs(qI).T) @ np.abs(hw)
    got = st.scores[s, :nv].double().cpu().numpy()
    floor = 1e-3 * float(np.max(np.abs(ref)))
    err = np.abs(got - ref) - bound
    assert np.all(err <= REL_TOL * np.maximum(np.abs(ref), floor)), err.max()

    # top-k set: complete, ascending, and equal to the oracle's except where
    # an entry's score is within the bounds of the k-th score
    gi = st.idx[s].cpu().numpy()
    assert np.all(gi >= 0) and np.all(np.diff(gi) > 0) and len(gi) == k
    order = np.argsort(-ref, kind="stable")
    kth, bk = ref[order[k - 1]], bound[order[k - 1]]
    band = GAP_TOL + bk + bound
    sel = set(gi.tolist())
    assert set(np.nonzero(ref > kth + band)[0].tolist()) <= sel
    assert not (sel & set(np.nonzero(ref < kth - band)[0].tolist()))

    # attention over the GPU's selected set (oracle rows from the raw streams) + window
    rows = []
    for e in gi:
        c, _ = oracle.gate_pool(kv[e * m:(e + 1) * m], wg, gb)
        r, sc = oracle.quantize(oracle.rope(oracle.rmsnorm(c, gamma_kv, 1e-6), int(e) * m, 10000.0, 64), 64)
        rows.append(oracle.dequantize(r, sc, D))
    for p in range(Ls - 128, Ls):
        r, sc = oracle.window_row(kv[p], gamma_kv, p)
        rows.append(oracle.dequantize(r, sc, D))
    out, _ = oracle.attend(q, gamma_q, Ls - 1, np.stack(rows), sink)
    gout = st.out[s].double().cpu().numpy()
    e = np.abs(gout - out)
    rms = math.sqrt(float(np.mean(out * out)))
    assert e.max() <= MAX_ABS and e.max() <= 2e-2 * rms, (e.max(), rms)
