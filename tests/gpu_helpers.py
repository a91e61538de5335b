"""GPU-side test assembly: layers built through the library's own
csla_compress_append from the seeded token streams, plus comparison helpers
that classify quantised codes against the oracle's decision values."""
import numpy as np
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import CompressParams, LayerBuffers, LayerShape
from csla_synth.workloads import Workload, layer_params, token_stream
from helpers import block_table

DEV = "cuda"


def shape_of(w: Workload):
    return LayerShape(m=w.m, D=w.D, H=w.H, HI=w.HI or 16, dI=w.dI or 128, dc=w.dc or 1024, n_win=w.n_win,
                      d_rope=w.d_rope, theta=w.theta, eps=w.eps, key_fmt=w.key_fmt, gate=w.gate)


def act_tensor(w: Workload, x):
    t = torch.as_tensor(np.ascontiguousarray(x), dtype=torch.float64)
    return t.to(torch.bfloat16 if w.act_bf16 else torch.float32).to(DEV).contiguous()


def build_layer(w: Workload, lens, params=None, chunk=None, extra_pages=0):
    """Append every request's stream 0..L-1 through csla_compress_append
    (`chunk` tokens per call; None = one call per request)."""
    p = params or layer_params(w)
    shape = shape_of(w)
    bt, n_pages = block_table(w, lens, len(lens))
    lb = LayerBuffers(shape, len(lens), n_pages + extra_pages, bt.shape[1], DEV)
    lb.block_table.copy_(torch.from_numpy(bt))
    cp = CompressParams(p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"), p.get("gbi"), DEV)
    for s, L in enumerate(lens):
        ts = token_stream(w, s, 0, L)
        append(w, lb, cp, s, ts, 0, L, chunk)
    torch.cuda.synchronize()
    return lb, cp, p


def append(w, lb, cp, slot, ts, start, stop, chunk=None):
    step = (stop - start) if chunk is None else chunk
    slots = torch.tensor([slot], dtype=torch.int32, device=DEV)
    for a in range(start, stop, step):
        b = min(stop, a + step)
        kv = act_tensor(w, ts["kv"][a - start:b - start])
        ki = act_tensor(w, ts["idx"][a - start:b - start]) if w.is_csa else None
        C.csla_compress_append(lb.cfg(), lb.state(), lb.cache(), slots, 1, b - a, kv, ki,
                               C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32, cp.struct())


def upload_layer(w: Workload, cv, lens):
    """Device copy of a cache the oracle built (tests/helpers.oracle_cache):
    the GPU steps then read exactly the bytes the oracle decodes."""
    n_pages = cv.rows.shape[0]
    lb = LayerBuffers(shape_of(w), len(lens), n_pages, cv.block_table.shape[1], DEV)
    fill_layer(lb, w, cv, lens)
    return lb


def fill_layer(lb: LayerBuffers, w: Workload, cv, lens, stream_ids=None):
    """Copy an oracle-built cache into existing layer buffers (the block
    table too: with a table shared by several layers it must be the same),
    and put the raw rows of every request's open block into the tail, so
    that the next appends close blocks from the right rows."""
    lb.rows.copy_(torch.from_numpy(cv.rows))
    lb.scales.copy_(torch.from_numpy(cv.scales))
    if w.is_csa and cv.kscale is not None:
        lb.kidx.copy_(torch.from_numpy(cv.kidx))
        lb.kscale.copy_(torch.from_numpy(cv.kscale))
    elif w.is_csa:
        lb.kidx.copy_(torch.from_numpy(cv.kidx.view(np.int16)))
    lb.block_table.copy_(torch.from_numpy(cv.block_table))
    lb.win_rows.copy_(torch.from_numpy(cv.win_rows))
    lb.win_scales.copy_(torch.from_numpy(cv.win_scales))
    lb.len.copy_(torch.tensor(list(lens), dtype=torch.int32))
    for slot, L in enumerate(lens):
        n = int(L) % w.m
        if n:
            ts = token_stream(w, slot if stream_ids is None else stream_ids[slot], int(L) - n, int(L))
            lb.tail_kv[slot, :n] = torch.from_numpy(ts["kv"].astype(np.float32))
            if w.is_csa:
                lb.tail_idx[slot, :n] = torch.from_numpy(ts["idx"].astype(np.float32))
    torch.cuda.synchronize()


def cache_view(w: Workload, lb: LayerBuffers):
    h = lb.host_view()
    return oracle.CacheView(w.m, w.D, h["rows"], h["scales"], h["block_table"], h["win_rows"],
                            h["win_scales"], h.get("kidx"), w.dI, w.d_rope, kscale=h.get("kscale"))


def assert_no_device_error():
    rc, bits = C.csla_device_error()
    assert rc == C.CSLA_OK, "device error bits 0x%x" % bits


_E4M3 = np.array([oracle.e4m3_value(c) for c in range(128)])
_E4M3_FINITE = np.sort(_E4M3[np.isfinite(_E4M3)])
_MIDS = 0.5 * (_E4M3_FINITE[1:] + _E4M3_FINITE[:-1])


def near_midpoint(v, rel=1e-5):
    """True where |v| lies within `rel` of an E4M3 rounding midpoint."""
    a = np.abs(np.asarray(v, np.float64))
    i = np.clip(np.searchsorted(_MIDS, a), 1, len(_MIDS) - 1)
    d = np.minimum(np.abs(a - _MIDS[i - 1]), np.abs(a - _MIDS[i]))
    return d <= rel * np.maximum(a, 2.0 ** -9)


def compare_rows(gpu_row, gpu_scale, y, D, d_rope=64):
    """Compare one GPU cache row with the oracle's fp64 pre-quantisation
    vector y.  Both sides quantise in fp32: codes must match exactly except
    where the oracle's fp32 value y/scale is within 1e-5 of a rounding
    midpoint (then one step either way is allowed); the scale must agree to
    fp32 rounding of amax; the bf16 RoPE dims must match except at a bf16
    rounding tie.  Returns the number of tolerated code differences."""
    dn = D - d_rope
    ref_row, ref_scale = oracle.quantize(y, d_rope)
    assert abs(float(gpu_scale) - float(ref_scale)) <= 2e-6 * abs(float(ref_scale)), (gpu_scale, ref_scale)
    v = (np.asarray(y[:dn], np.float64).astype(np.float32) / np.float32(ref_scale)).astype(np.float64)
    g = np.asarray(gpu_row[:dn], np.uint8)
    r = np.asarray(ref_row[:dn], np.uint8)
    diff = np.nonzero(g != r)[0]
    for d in diff:
        assert near_midpoint(v[d]), ("code mismatch", d, hex(g[d]), hex(r[d]), v[d])
        gv, rv = _E4M3[g[d] & 0x7F], _E4M3[r[d] & 0x7F]
        # adjacent representable values
        gi, ri = np.searchsorted(_E4M3_FINITE, gv), np.searchsorted(_E4M3_FINITE, rv)
        assert abs(int(gi) - int(ri)) <= 1
    gr = np.asarray(gpu_row[dn:], np.uint8).view(np.uint16)
    rr = np.asarray(ref_row[dn:], np.uint8).view(np.uint16)
    assert_bf16_close(gr, rr, 1e-6 * float(np.max(np.abs(y))))
    return len(diff)


def bf16_values(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_bf16_close(got_bits, ref_bits, abs_tol):
    """bf16 results of a float computation done in fp32 (GPU) and fp64
    (oracle): each side rounds its own value once, so they may differ by one
    bf16 ulp at the larger magnitude, plus the fp32 arithmetic error abs_tol
    (which matters where terms cancel and the result is near zero, where a
    bit-pattern distance would be meaningless, e.g. across a sign change)."""
    g, r = bf16_values(got_bits), bf16_values(ref_bits)
    mag = np.maximum(np.abs(g), np.abs(r))
    ulp = np.exp2(np.floor(np.log2(np.maximum(mag, 1e-38))) - 7)
    bad = np.nonzero(np.abs(g - r) > ulp + abs_tol)[0]
    assert len(bad) == 0, [(int(i), g[i], r[i]) for i in bad[:8]]


MAX_ABS = 1e-2        # attention: the contract's bound for O(1) outputs
REL_RMS = 2e-2        # attention: derived bound, error / RMS(output) (f16/bf16 q and P operands)
REL_TOL = 1e-3        # indexer scores, relative to max(|oracle|, 1e-3 * row max)


def check_out(got, ref):
    """Attention output of one request against the oracle's fp64 result."""
    err = np.abs(got - ref)
    rms = np.sqrt(np.mean(ref * ref))
    assert np.all(np.isfinite(got))
    assert err.max() <= MAX_ABS, err.max()
    assert err.max() <= REL_RMS * rms, (err.max(), rms)
    return err.max()


def check_scores(got, ref):
    """Indexer scores of one request against the oracle's fp64 scores."""
    floor = 1e-3 * max(np.max(np.abs(ref)), 1e-30)
    err = np.abs(got - ref) / np.maximum(np.abs(ref), floor)
    assert np.all(np.isfinite(got))
    assert err.max() <= REL_TOL, err.max()
    return err.max()


def check_csa_step(w: Workload, cv, p, si, lens, gidx, gout):
    """One CSA decode step of len(lens) requests on the GPU (top-k lists
    gidx, outputs gout) against the oracle on the cache cv: every entry
    scoring clearly above the k-th oracle score is selected, none clearly
    below; the output matches the oracle's step, or, where a tie inside the
    band picked another set, the oracle's attention over the GPU's set."""
    B = len(lens)
    oidx, oout = oracle.csa_decode(cv, np.arange(B), lens, si["q"][:B], p["gamma_q"], si["cq"][:B], p["W_iq"],
                                   si["head_w"][:B], p["sink"], w.HI, w.k, w.eps, w.theta)
    for s, L in enumerate(lens):
        nv = L // w.m
        sel = set(int(x) for x in gidx[s] if x >= 0)
        if nv > 0:
            qI = oracle.index_query(si["cq"][s], p["W_iq"], w.HI, w.dI)
            ref = oracle.index_scores(qI, si["head_w"][s], cv.gather_keys(s, nv))
            kth = np.sort(ref)[::-1][min(w.k, nv) - 1]
            assert set(np.nonzero(ref > kth + 1e-4)[0].tolist()) <= sel, s
            assert not (sel & set(np.nonzero(ref < kth - 1e-4)[0].tolist())), s
        if set(oidx[s][oidx[s] >= 0].tolist()) == sel:
            check_out(gout[s], oout[s])
        else:
            rows = cv.gather_set(s, L, gidx[s])
            r2, _ = oracle.attend(si["q"][s], p["gamma_q"], L - 1, rows, p["sink"], w.eps, w.theta, w.d_rope)
            check_out(gout[s], r2)
