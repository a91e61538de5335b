"""The multi-GPU path is data parallel over requests (weak scaling, no
collective on the data path): world-size-2 gloo runs on CPU check its host
side -- the job's step time is the max over ranks (bench.dp_max), and a
request's result does not depend on which rank serves it or with whom (each
rank runs the oracle on its own shard; the gathered results equal one
single-process run bit for bit)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

WORLD = 2
GLOBAL_B = 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _decode(ids):
    """Oracle CSA decode (tiny config) of the global requests `ids`, each in
    its own cache slot, with per-request inputs taken by global id."""
    import dataclasses
    import oracle
    from csla_synth.workloads import CSA_TINY, step_inputs
    from helpers import oracle_cache
    w = dataclasses.replace(CSA_TINY, B=GLOBAL_B, L=700, name="dp_gloo")
    lens = [700 - 37 * g for g in range(GLOBAL_B)]
    cv, p = oracle_cache(w, [lens[g] for g in ids], stream_ids=ids)
    si = step_inputs(w, 3)
    sel = np.asarray(ids)
    idx, out = oracle.csa_decode(cv, list(range(len(ids))), [lens[g] for g in ids], si["q"][sel],
                                 p["gamma_q"], si["cq"][sel], p["W_iq"], si["head_w"][sel], p["sink"], w.HI, w.k)
    return idx, out


def _rank_main(rank, port, ret):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=timedelta(seconds=60))
    try:
        import bench
        # step time of the job = slowest rank
        got = bench.dp_max([1.25, 2.5][rank], WORLD, torch.device("cpu"))
        assert got == 2.5, got
        # rank r serves global requests r*2, r*2+1
        ids = [rank * (GLOBAL_B // WORLD) + i for i in range(GLOBAL_B // WORLD)]
        idx, out = _decode(ids)
        gathered = [None] * WORLD
        dist.all_gather_object(gathered, (ids, idx, out))
        if rank == 0:
            all_ids = sum((g[0] for g in gathered), [])
            assert sorted(all_ids) == list(range(GLOBAL_B))
            ref_idx, ref_out = _decode(list(range(GLOBAL_B)))
            for ids_r, idx_r, out_r in gathered:
                for i, g in enumerate(ids_r):
                    assert np.array_equal(idx_r[i], ref_idx[g])
                    assert np.array_equal(out_r[i], ref_out[g])
            ret.put("ok")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_dp_over_requests_world2_gloo():
    import oracle
    oracle.lib()   # build (if needed) once, before the ranks load it
    ctx = mp.get_context("spawn")
    ret = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(_free_port(), ret), nprocs=WORLD, join=True, start_method="spawn")
    assert ret.get() == "ok"
