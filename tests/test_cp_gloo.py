"""Context-parallel prefill, host side, on CPU ranks (gloo): the plan's
bookkeeping and the distributed driver (boundary send/recv, all-gather of
padded entry runs, reassembly by global block index) with each rank's
compute done by the oracle.  Every rank must end with the compressed cache
of the whole request, byte for byte the single-process oracle's, and the
window rows of its own queries.  The entry record is the library's
(include/csla.h: row | key | f32 scale | f32 key scale | zero pad to 16)."""
import dataclasses
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from compressed_sparse_long_append_b200.cp import cp_plan, run_cp_prefill


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(kind):
    from csla_synth.workloads import CSA_DECODE, CSA_TINY, HCA_DECODE
    if kind == "csa":
        return dataclasses.replace(CSA_TINY, B=1, L=1500, name="cp_csa")
    if kind == "csa_e4m3_channel":
        return dataclasses.replace(CSA_DECODE, B=1, L=1500, H=8, key_fmt=1, gate=1, name="cp_csa8")
    return dataclasses.replace(HCA_DECODE, B=1, L=1300, H=8, name="cp_hca")


def _key_bytes(w):
    if not w.is_csa:
        return 0
    return w.dI if w.key_fmt == 1 else 2 * w.dI


def _rec_bytes(w):
    import oracle
    return (oracle.row_bytes(w.D, w.d_rope) + _key_bytes(w) + 8 + 15) // 16 * 16


def _expected(w, p, kv, ki, L0, L1):
    import oracle
    return oracle.expected_append(kv, ki, L0, L1, w.m, p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"),
                                  p.get("gbi"), w.eps, w.theta, w.d_rope, window_from=L0,
                                  key_e4m3=w.key_fmt == 1, per_channel=w.gate == 1)


def _key_to_bytes(w, key):
    if w.key_fmt == 1:
        codes, ks = key
        return np.asarray(codes, np.uint8).tobytes(), float(ks)
    return np.asarray(key, np.uint16).tobytes(), 0.0


class OracleRank:
    """Rank r's steps done by the oracle on host arrays.  Rows the rank never
    received stay NaN, so a wrong boundary shows up in the results."""

    def __init__(self, plan, r, w, p):
        self.plan, self.r, self.w, self.p = plan, r, w, p
        N = plan.N
        self.kv = np.full((N, w.D), np.nan)
        self.ki = np.full((N, w.dI), np.nan) if w.is_csa else None
        self.cache, self.win = {}, {}

    def boundary_out(self, kv, kidx=None):
        a = self.plan.bnd_offset(self.r)
        return kv[a:], (kidx[a:] if kidx is not None else None)

    def compress(self, bkv, bki, kv, kidx):
        plan, r = self.plan, self.r
        a, (p0, p1) = plan.bnd_start(r), plan.rng(r)
        if bkv is not None:
            self.kv[a:p0] = bkv.numpy()
            if self.ki is not None:
                self.ki[a:p0] = bki.numpy()
        self.kv[p0:p1] = kv.numpy()
        if self.ki is not None:
            self.ki[p0:p1] = kidx.numpy()
        exp = _expected(self.w, self.p, self.kv, self.ki, a, p1)
        for b, (row, sc) in exp["entries"].items():
            self.cache[b] = (np.asarray(row, np.uint8).tobytes(), float(sc),
                             _key_to_bytes(self.w, exp["keys"][b]) if self.w.is_csa else (b"", 0.0))
        self.win.update({pos: (np.asarray(rw, np.uint8).tobytes(), float(sc)) for pos, (rw, sc) in
                         exp["window"].items()})

    def select(self):
        b_lo, n = self.plan.blocks(self.r)
        rec = _rec_bytes(self.w)
        out = np.zeros((self.plan.E_max, rec), np.uint8)
        for j in range(n):
            row, sc, (key, ks) = self.cache[b_lo + j]
            tail = np.array([sc, ks], np.float32).tobytes()
            blob = row + key + tail
            out[j, :len(blob)] = np.frombuffer(blob, np.uint8)
        return torch.from_numpy(out)

    def place(self, recv):
        import oracle
        rb = oracle.row_bytes(self.w.D, self.w.d_rope)
        kb = _key_bytes(self.w)
        recv = recv.numpy()
        for q in range(self.plan.R):
            b_lo, n = self.plan.blocks(q)
            for j in range(n):
                rec = recv[q, j]
                row = rec[:rb].tobytes()
                key = rec[rb:rb + kb].tobytes()
                sc, ks = np.frombuffer(rec[rb + kb:rb + kb + 8].tobytes(), np.float32)
                self.cache[b_lo + j] = (row, float(sc), (key, float(ks)))


def _inputs(w, N):
    from csla_synth.workloads import token_stream
    ts = token_stream(w, 0, 0, N)
    return ts["kv"], ts.get("idx")


def _rank_main(rank, world, port, kind, starts, ret):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from csla_synth.workloads import layer_params
        w = _workload(kind)
        p = layer_params(w)
        N = w.L
        plan = cp_plan(N, world, w.m, w.n_win, starts=starts)
        kv, ki = _inputs(w, N)
        p0, p1 = plan.rng(rank)
        obj = OracleRank(plan, rank, w, p)
        run_cp_prefill(obj, torch.from_numpy(kv[p0:p1].copy()),
                       torch.from_numpy(ki[p0:p1].copy()) if ki is not None else None)
        # the whole request's cache, as one process computes it
        full = _expected(w, p, kv, ki, 0, N)
        assert sorted(obj.cache) == list(range(N // w.m)), (rank, sorted(obj.cache)[:5])
        for b, (row, sc) in full["entries"].items():
            grow, gsc, (gkey, gks) = obj.cache[b]
            assert grow == np.asarray(row, np.uint8).tobytes() and np.float32(gsc) == np.float32(sc), (rank, b)
            if w.is_csa:
                key, ks = _key_to_bytes(w, full["keys"][b])
                assert gkey == key and np.float32(gks) == np.float32(ks), (rank, b)
        # window rows of this rank's queries: positions p0-127 .. p1-1
        for pos in range(max(0, p0 - (w.n_win - 1)), p1):
            row, sc = full["window"][pos]
            assert obj.win[pos][0] == np.asarray(row, np.uint8).tobytes() and \
                np.float32(obj.win[pos][1]) == np.float32(sc), (rank, pos)
        ret[rank] = "ok"
    except Exception as e:  # reported by the parent
        import traceback
        ret[rank] = traceback.format_exc()
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind,world,starts", [
    ("csa", 2, None),
    ("csa", 3, [0, 400, 1001, 1500]),             # uneven, boundaries mid-block
    ("csa_e4m3_channel", 2, [0, 733, 1500]),       # E4M3 keys, per-channel gate
    ("hca", 2, [0, 645, 1300]),                    # HCA: a 128-token block across the boundary
    ("hca", 3, [0, 300, 811, 1300]),
    ("csa", 4, [0, 300, 640, 1003, 1500]),        # boundary exactly at a page start (640)
    ("hca", 4, [0, 256, 512, 1024, 1300]),         # boundaries at block starts: no open block to send
])
def test_cp_prefill_on_gloo_ranks(kind, world, starts):
    port = _free_port()
    with mp.Manager() as mgr:
        ret = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, kind, starts, ret), nprocs=world, join=True)
        for r in range(world):
            assert ret.get(r) == "ok", ret.get(r)


def test_cp_plan_bookkeeping():
    plan = cp_plan(1500, 3, 4, 128, starts=[0, 400, 1001, 1500])
    assert plan.blocks(0) == (0, 100) and plan.blocks(1) == (100, 150) and plan.blocks(2) == (250, 125)
    assert sum(plan.blocks(r)[1] for r in range(3)) == 1500 // 4 and plan.E_max == 150
    # boundary: block-aligned, covers the 127 window positions and the open block
    for r in (1, 2):
        a, p = plan.bnd_start(r), plan.starts[r]
        assert a % 4 == 0 and p - a >= 127 and a // 4 == (p - 127) // 4 and p - a <= plan.head_rows
    hca = cp_plan(1300, 3, 128, 128, starts=[0, 300, 811, 1300])
    assert hca.bnd_start(1) == 128 and hca.bnd_start(2) == 640 and hca.n_bnd(2) == 171 <= hca.head_rows
    assert [hca.blocks(r) for r in range(3)] == [(0, 2), (2, 4), (6, 4)]
    with pytest.raises(ValueError):
        cp_plan(1300, 3, 128, 128, starts=[0, 300, 400, 1300])   # rank 1 shorter than rank 2's boundary
    with pytest.raises(ValueError):
        cp_plan(100, 2, 4, 128, starts=[0, 0, 100])
