"""The allocation-free indexer entry point (csla_indexer_scores_noalloc).

It exists for callers that cannot call cudaMalloc -- a framework that has
reserved the whole device pool, code running in an allocator hook or host
callback -- and so cannot provide the indexer's workspace.  The test calls
it twice in a row through the C ABI (the second call with new query-side
inputs, so stale scratch from the first call would show) and compares each
result with the regular entry point's.  Both launch the same kernels on the
same inputs, only the scratch address differs, so the scores must agree bit
for bit.  It is
collected last so that a failure here never hides the other tests.
"""
import dataclasses

import numpy as np
import pytest
import torch

from compressed_sparse_long_append_b200 import csla as C
from csla_synth.workloads import CSA_DECODE, CSA_TINY, step_inputs
from gpu_helpers import DEV, act_tensor, assert_no_device_error, upload_layer
from helpers import oracle_cache

pytestmark = pytest.mark.gpu


def _scores(w, lb, si, p, lens, noalloc):
    B, max_len = len(lens), max(lens)
    stride = max_len // w.m
    out = torch.full((B, stride), float("nan"), dtype=torch.float32, device=DEV)
    slots = torch.arange(B, dtype=torch.int32, device=DEV)
    cq, W = act_tensor(w, si["cq"][:B]), act_tensor(w, p["W_iq"])
    hw = torch.as_tensor(si["head_w"][:B], dtype=torch.float32, device=DEV)
    dt = C.CSLA_BF16 if w.act_bf16 else C.CSLA_F32
    if noalloc:
        C.csla_indexer_scores_noalloc(lb.cfg(), lb.state(), lb.cache(), slots, B, max_len, cq, dt, W, dt, hw,
                                      out, stride)
    else:
        wsb = C.csla_workspace_size(lb.cfg(), C.CSLA_OP_INDEXER, B, max_len)
        ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
        C.csla_indexer_scores(lb.cfg(), lb.state(), lb.cache(), slots, B, max_len, cq, dt, W, dt, hw, out,
                              stride, ws, wsb)
    assert_no_device_error()
    return out.cpu().numpy()


@pytest.mark.parametrize("w,lens", [
    (dataclasses.replace(CSA_TINY, B=2, L=1500, name="noalloc_tiny"), [1500, 401]),
    (dataclasses.replace(CSA_DECODE, B=3, L=3000, name="noalloc_big"), [3000, 2222, 513]),
])
def test_noalloc_indexer_matches_regular_entry_point(w, lens):
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    for call in range(2):                      # two calls in a row, different inputs
        si = step_inputs(w, 20 + call)
        ref = _scores(w, lb, si, p, lens, noalloc=False)
        got = _scores(w, lb, si, p, lens, noalloc=True)
        for s, L in enumerate(lens):
            nv = L // w.m
            assert np.array_equal(got[s, :nv], ref[s, :nv])
            assert np.all(np.isnan(got[s, nv:]))


def test_noalloc_rejects_batches_beyond_its_scratch():
    w = dataclasses.replace(CSA_DECODE, B=1, L=600, name="noalloc_limit")
    lens = [600]
    cv, p = oracle_cache(w, lens)
    lb = upload_layer(w, cv, lens)
    per_request = 48 * 128 * 2
    too_many = C.CSLA_NOALLOC_INDEXER_SCRATCH_BYTES // per_request + 1
    dummy = torch.zeros(16, dtype=torch.float32, device=DEV)
    rc = C._lib.csla_indexer_scores_noalloc(
        C.ctypes.byref(lb.cfg()), C.ctypes.byref(lb.state()), C.ctypes.byref(lb.cache()), dummy.data_ptr(),
        too_many, None, 600, dummy.data_ptr(), C.CSLA_BF16, dummy.data_ptr(), C.CSLA_BF16, dummy.data_ptr(),
        dummy.data_ptr(), 150, torch.cuda.current_stream().cuda_stream)
    assert rc == C.CSLA_ERR_ARG
