"""A model-shaped stack of emulated attention layers on one block table:
CSA and HCA layers interleaved (the hybrid configuration of the source
pages, read as strict alternation), each layer with its own parameters,
pools, window ring and tail, every layer's cache paged through the SAME
per-request table of 128-token pages.  Decode steps through the library,
layer after layer; after every step each layer's output and length are
checked against the oracle run on that layer alone."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_append_b200 import csla as C
from compressed_sparse_long_append_b200.layer import CompressParams, LayerStack
from csla_synth.workloads import CSA_DECODE, CSA_TINY, HCA_DECODE, step_inputs, token_stream
from gpu_helpers import DEV, act_tensor, assert_no_device_error, check_csa_step, check_out, fill_layer, shape_of
from helpers import block_table, oracle_cache

pytestmark = pytest.mark.gpu


def _f32(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float32, device=DEV)


def _stack(B):
    """Four layers: CSA (per-channel gate), HCA, CSA (E4M3 index keys), HCA
    (per-channel gate); one shape family per kind, a seed per layer."""
    csa = dataclasses.replace(CSA_DECODE, B=B, L=0, H=16, k=64)
    hca = dataclasses.replace(HCA_DECODE, B=B, L=0, H=16)
    return [dataclasses.replace(csa, seed=30, gate=1, name="stack0"),
            dataclasses.replace(hca, seed=31, name="stack1"),
            dataclasses.replace(csa, seed=32, key_fmt=1, name="stack2"),
            dataclasses.replace(hca, seed=33, gate=1, name="stack3")]


def test_interleaved_stack_on_one_block_table():
    lens0 = [1100, 385, 7]
    B, n_steps = len(lens0), 3
    layers = _stack(B)
    bt, n_pages = block_table(layers[0], [L + n_steps for L in lens0], B, seed_name="stack_bt")
    stack = LayerStack([shape_of(w) for w in layers], B, n_pages, bt.shape[1], DEV)
    stack.block_table.copy_(torch.from_numpy(bt))
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    max_len = max(lens0) + n_steps
    state = []
    for i, w in enumerate(layers):
        cv, p = oracle_cache(w, lens0, bt=bt)
        lb = stack.layers[i]
        fill_layer(lb, w, cv, lens0)   # rewrites the shared table with the same content
        st = {"p": p, "cp": CompressParams(p["gamma_kv"], p["wg"], p["gb"], p.get("wgi"), p.get("gbi"), DEV),
              "out": torch.full((B, w.H, w.D), float("nan"), dtype=torch.float32, device=DEV)}
        cfg = lb.cfg()
        if w.is_csa:
            st["stride"] = max_len // w.m
            st["scores"] = torch.zeros((B, st["stride"]), dtype=torch.float32, device=DEV)
            st["idx"] = torch.full((B, w.k), -7, dtype=torch.int32, device=DEV)
            st["wsi_b"] = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, max_len)
            st["wss_b"] = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_DECODE_STEP, B, w.k)
            st["wsi"] = torch.zeros(st["wsi_b"], dtype=torch.uint8, device=DEV)
            st["wss"] = torch.zeros(st["wss_b"], dtype=torch.uint8, device=DEV)
            st["W"] = act_tensor(w, p["W_iq"])
        else:
            st["wsa_b"] = C.csla_workspace_size(cfg, C.CSLA_OP_HCA_ATTEND, B, max_len)
            st["wsa"] = torch.zeros(st["wsa_b"], dtype=torch.uint8, device=DEV)
        state.append(st)
    torch.cuda.synchronize()
    # every layer's cache struct names the one table
    assert len({lb.cache().block_table for lb in stack.layers}) == 1

    dt = C.CSLA_BF16
    for step in range(n_steps):
        lens = [L + step + 1 for L in lens0]
        sis = []
        for i, w in enumerate(layers):   # layer after layer, as a model's decode step runs them
            lb, st = stack.layers[i], state[i]
            si = step_inputs(w, 70 + step)
            sis.append(si)
            kv = act_tensor(w, np.stack([token_stream(w, b, L - 1, L)["kv"] for b, L in enumerate(lens)]))
            q = act_tensor(w, si["q"][:B])
            sink, gq = _f32(st["p"]["sink"]), _f32(st["p"]["gamma_q"])
            if w.is_csa:
                ki = act_tensor(w, np.stack([token_stream(w, b, L - 1, L)["idx"] for b, L in enumerate(lens)]))
                C.csla_csa_decode_step(lb.cfg(), lb.state(), lb.cache(), slots, B, 1, max_len, kv, ki, dt,
                                       st["cp"].struct(), act_tensor(w, si["cq"][:B]), dt, st["W"], dt,
                                       _f32(si["head_w"][:B]), st["scores"], st["stride"], w.k, st["idx"], q, dt,
                                       sink, gq, st["out"], C.CSLA_F32, C.CSLA_VARIANT_AUTO, st["wsi"],
                                       st["wsi_b"], st["wss"], st["wss_b"])
            else:
                C.csla_compress_append(lb.cfg(), lb.state(), lb.cache(), slots, B, 1, kv, None, dt,
                                       st["cp"].struct())
                C.csla_hca_attend(lb.cfg(), lb.state(), lb.cache(), slots, B, max_len, q, dt, sink, gq,
                                  st["out"], C.CSLA_F32, C.CSLA_VARIANT_AUTO, st["wsa"], st["wsa_b"])
        assert_no_device_error()
        for i, w in enumerate(layers):
            lb, st, si = stack.layers[i], state[i], sis[i]
            assert lb.len.cpu().tolist() == lens, (step, i)
            cv, p = oracle_cache(w, lens, bt=bt)
            got = st["out"].cpu().numpy().astype(np.float64)
            assert np.all(np.isfinite(got)), (step, i)
            try:
                if w.is_csa:
                    check_csa_step(w, cv, p, si, lens, st["idx"].cpu().numpy(), got)
                else:
                    ref = oracle.hca_decode(cv, np.arange(B), lens, si["q"][:B], p["gamma_q"], p["sink"], w.eps,
                                            w.theta)
                    for s in range(B):
                        check_out(got[s], ref[s])
            except AssertionError as e:
                raise AssertionError("step %d layer %d (%s): %s" % (step, i, w.name, e)) from None
    # the table itself is only read
    assert np.array_equal(stack.block_table.cpu().numpy(), bt)
