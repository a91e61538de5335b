"""CPU checks of the C ABI: libcsla.so loads without a GPU, exports every
entry point include/csla.h declares, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "csla.h")


def declared(timeline=False):
    """Entry points the header declares for a normal build (the device
    timeline readers exist only in builds with -DCSLA_TIMELINE)."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    if not timeline:
        txt = re.sub(r"#ifdef CSLA_TIMELINE.*?#endif", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(csla_[a-z_]+)\s*\(", txt)))


def test_timeline_readers_are_build_variant_only():
    from compressed_sparse_long_append_b200 import csla
    lib = ctypes.CDLL(csla.LIB_PATH)
    extra = set(declared(timeline=True)) - set(declared())
    assert extra == {"csla_timeline_read", "csla_timeline_clear"}
    for n in extra:
        assert not hasattr(lib, n), n


def test_header_declares_the_five_calls():
    names = declared()
    for n in ("csla_compress_append", "csla_indexer_scores", "csla_topk_select", "csla_csa_attend",
              "csla_hca_attend", "csla_workspace_size", "csla_device_error", "csla_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from compressed_sparse_long_append_b200 import csla
    lib = ctypes.CDLL(csla.LIB_PATH)
    for n in declared():
        assert hasattr(lib, n), n
    assert set(csla.EXPORTS) <= set(declared())


def _cfg(**kw):
    from compressed_sparse_long_append_b200.layer import LayerShape
    return LayerShape(**kw).cfg()


def test_host_argument_checks():
    from compressed_sparse_long_append_b200 import csla as C
    L = C._lib
    cfg = _cfg(m=4)
    # null structs / pointers -> CSLA_ERR_ARG, no launch
    assert L.csla_compress_append(ctypes.byref(cfg), None, None, None, 1, 1, None, None, 0, None, None,
                                  None) == C.CSLA_ERR_ARG
    assert L.csla_topk_select(ctypes.byref(cfg), None, None, 1, None, 10, None, 10, 5, None, None) == C.CSLA_ERR_ARG
    assert L.csla_hca_attend(ctypes.byref(_cfg(m=128)), None, None, None, 1, None, 100, None, 0, None, None, None,
                             0, 0, None, 0, None) == C.CSLA_ERR_ARG
    assert L.csla_window_rows(ctypes.byref(cfg), None, None, 1, 127, None, None, 127, None) == C.CSLA_ERR_ARG
    # query rows without q_len, or a window source without its bases -> CSLA_ERR_ARG before any launch
    fake = 1 << 40   # never dereferenced: the host check fails first
    st = C.csla_state(fake, fake, fake, fake, fake, 4)
    no_len = C.csla_queries(None, None, None, None, 0)
    assert L.csla_topk_select(ctypes.byref(cfg), ctypes.byref(st), fake, 1, ctypes.byref(no_len), 10, fake, 10, 5,
                              fake, None) == C.CSLA_ERR_ARG
    no_base = C.csla_queries(fake, fake, fake, None, 10)
    assert L.csla_topk_select(ctypes.byref(cfg), ctypes.byref(st), fake, 1, ctypes.byref(no_base), 10, fake, 10, 5,
                              fake, None) == C.CSLA_ERR_ARG
    # unsupported shapes
    for bad in (dict(m=8), dict(m=4, D=256), dict(m=4, d_rope=32), dict(m=4, H=65), dict(m=4, n_win=64)):
        assert L.csla_topk_select(ctypes.byref(_cfg(**bad)), None, None, 1, None, 10, None, 10, 5, None, None) \
            == C.CSLA_ERR_UNSUPPORTED, bad
    assert L.csla_topk_select(ctypes.byref(_cfg(m=4, gate=2)), None, None, 1, None, 10, None, 10, 5, None, None) \
        == C.CSLA_ERR_UNSUPPORTED
    # per-channel gate biases must be 16-byte aligned
    cst = C.csla_state(fake, fake, fake, fake, fake, 4)
    cch = C.csla_cache(fake, fake, fake, fake, 8, 16)
    odd = C.csla_compress_params(fake, fake, fake + 4, fake, fake)
    assert L.csla_compress_append(ctypes.byref(_cfg(m=4, gate=C.CSLA_GATE_CHANNEL)), ctypes.byref(cst),
                                  ctypes.byref(cch), fake, 1, 1, fake, fake, C.CSLA_BF16, ctypes.byref(odd), None,
                                  None) == C.CSLA_ERR_ARG
    assert L.csla_strerror(C.CSLA_ERR_DEVICE) == b"device-side input error"
    # the bounded-wait check takes 1 us .. 2 s
    assert L.csla_check_wait_timeout(0, None) == C.CSLA_ERR_ARG
    assert L.csla_check_wait_timeout(2000001, None) == C.CSLA_ERR_ARG
    # attention: row locations are 32-bit indices
    big = C.csla_cache(1 << 40, 1 << 40, None, 1 << 40, 1, 1 << 28)   # 2^28 pages x 32 entries = 2^33 rows
    stq = C.csla_state(1 << 40, 1 << 40, 1 << 40, 1 << 40, 1 << 40, 4)
    fake = 1 << 40
    assert L.csla_csa_attend(ctypes.byref(cfg), ctypes.byref(stq), ctypes.byref(big), fake, 1, None, fake,
                             C.CSLA_BF16, fake, 64, fake, fake, fake, C.CSLA_F32, 0, fake, 1 << 30, None) \
        == C.CSLA_ERR_UNSUPPORTED


def test_workspace_sizes():
    from compressed_sparse_long_append_b200 import csla as C
    cfg = _cfg(m=4)
    # indexer: B * NQ * dI bf16 with NQ = 3*HI rounded up to 16
    assert C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, 8, 131072) == 8 * 48 * 128 * 2
    assert C.csla_workspace_size(cfg, C.CSLA_OP_TOPK, 8, 131072) == 0
    # attention: B * chunks * (H*D + 2H) floats (chunk partials);
    # 512+128 rows -> 10 chunks of 64
    assert C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, 8, 512) == 8 * 10 * (64 * 512 + 128) * 4
    hca = _cfg(m=128)
    assert C.csla_workspace_size(hca, C.CSLA_OP_HCA_ATTEND, 4, 1 << 20) == 4 * 32 * (64 * 512 + 128) * 4
    assert C.csla_workspace_size(_cfg(m=8), C.CSLA_OP_TOPK, 1, 1) == 0
    # decode step: the attention partials for k, then B int32 lengths (16-byte rounded)
    assert C.csla_workspace_size(cfg, C.CSLA_OP_CSA_DECODE_STEP, 8, 512) == 8 * 10 * (64 * 512 + 128) * 4 + 32
    # indexer + top-k: the indexer's query terms, 1024 sample scores, a
    # threshold, four counts and a flag per row (int32, each part 16-byte
    # rounded), 8192 (key, entry) candidates per row
    assert C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER_TOPK, 8, 131072) == \
        8 * 48 * 128 * 2 + 8 * 1024 * 4 + 32 + 128 + 32 + 8 * 8192 * 8
    assert C.csla_workspace_size(_cfg(m=128), C.CSLA_OP_INDEXER_TOPK, 8, 131072) == 0
    # the binding's view of its parts agrees with the library's size
    for B, HI, dI in ((8, 16, 128), (37, 4, 64), (4096, 8, 128)):
        lay = C.indexer_topk_layout(B, HI, dI)
        assert lay["total"] == C.csla_workspace_size(_cfg(m=4, HI=HI, dI=dI), C.CSLA_OP_INDEXER_TOPK, B, 1 << 18)
        assert all(lay[k] % 16 == 0 for k in ("sample", "t0", "counts", "flags", "cand"))


def test_host_checks_of_the_query_row_and_step_calls():
    """Arguments the host rejects before any launch (no GPU needed)."""
    from compressed_sparse_long_append_b200 import csla as C
    L = C._lib
    fake = 1 << 40   # never dereferenced: every call below fails its host checks first
    cfg = _cfg(m=4)
    st = C.csla_state(fake, fake, fake, fake, fake, 4)
    cache = C.csla_cache(fake, fake, fake, fake, 8, 16)
    params = C.csla_compress_params(fake, fake, fake, fake, fake)
    # window snapshot: n outside 1..n_win, stride below n
    assert L.csla_window_rows(ctypes.byref(cfg), ctypes.byref(st), fake, 1, 129, fake, fake, 200, None) \
        == C.CSLA_ERR_ARG
    assert L.csla_window_rows(ctypes.byref(cfg), ctypes.byref(st), fake, 1, 100, fake, fake, 99, None) \
        == C.CSLA_ERR_ARG
    # token rows that do not fit the stride
    tok = C.csla_token_rows(fake, fake, 10, 5)
    assert L.csla_compress_append(ctypes.byref(cfg), ctypes.byref(st), ctypes.byref(cache), fake, 1, 6, fake, fake,
                                  C.CSLA_BF16, ctypes.byref(params), ctypes.byref(tok), None) == C.CSLA_ERR_ARG
    # the fused decode step: CSA only, and it needs a top-k list and its workspace
    args = [ctypes.byref(st), ctypes.byref(cache), fake, 1, 1, 1024, fake, fake, C.CSLA_BF16, ctypes.byref(params),
            fake, C.CSLA_BF16, fake, C.CSLA_BF16, fake, fake, 256, 64]
    tail = [fake, C.CSLA_BF16, fake, fake, fake, C.CSLA_F32, 0, fake, 1 << 20, fake, 1 << 20, None]
    assert L.csla_csa_decode_step(ctypes.byref(_cfg(m=128)), *args, fake, *tail) == C.CSLA_ERR_UNSUPPORTED
    assert L.csla_csa_decode_step(ctypes.byref(cfg), *args, None, *tail) == C.CSLA_ERR_ARG
    # indexer + top-k: k outside 1..2048, a workspace below its size, no scratch scores
    itk = [ctypes.byref(cfg), ctypes.byref(st), ctypes.byref(cache), fake, 8, None, 131072, fake, C.CSLA_BF16,
           fake, C.CSLA_BF16, fake]
    need = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER_TOPK, 8, 131072)
    assert L.csla_indexer_topk(*itk, 0, fake, fake, 32768, fake, need, None) == C.CSLA_ERR_ARG
    assert L.csla_indexer_topk(*itk, 2049, fake, fake, 32768, fake, need, None) == C.CSLA_ERR_ARG
    assert L.csla_indexer_topk(*itk, 1024, fake, fake, 32768, fake, need - 1, None) == C.CSLA_ERR_ARG
    assert L.csla_indexer_topk(*itk, 1024, fake, None, 32768, fake, need, None) == C.CSLA_ERR_ARG
    assert L.csla_indexer_topk(*itk, 1024, fake, fake, 1000, fake, need, None) == C.CSLA_ERR_ARG


def test_cp_record_size_and_host_checks():
    """Context-parallel entry records: size per the header's layout, and the
    arguments the host rejects before any launch."""
    from compressed_sparse_long_append_b200 import csla as C
    L = C._lib
    fake = 1 << 40
    # row 576 + bf16 key 256 + 8 -> 848; HCA row 576 + 8 -> 592; E4M3 key 128 -> 720
    assert C.csla_cp_record_bytes(_cfg(m=4)) == 848
    assert C.csla_cp_record_bytes(_cfg(m=128)) == 592
    assert C.csla_cp_record_bytes(_cfg(m=4, key_fmt=C.CSLA_KEY_E4M3)) == 720
    assert C.csla_cp_record_bytes(_cfg(m=4, D=128, dI=64)) == 192 + 128 + 16
    cfg = _cfg(m=4)
    st = C.csla_state(fake, fake, fake, fake, fake, 4)
    cache = C.csla_cache(fake, fake, fake, fake, 8, 16)
    arr = ctypes.c_int32 * 2
    sel = lambda slot, n, e, recs: L.csla_cp_select(ctypes.byref(cfg), ctypes.byref(st), ctypes.byref(cache), slot,
                                                    0, n, e, recs, None)
    assert sel(4, 1, 1, fake) == C.CSLA_ERR_ARG          # slot beyond the state's slots
    assert sel(0, 2, 1, fake) == C.CSLA_ERR_ARG          # more records than the run holds
    assert sel(0, 1, 1, fake + 8) == C.CSLA_ERR_ARG      # misaligned records
    place = lambda R, b, n: L.csla_cp_place(ctypes.byref(cfg), ctypes.byref(st), ctypes.byref(cache), 0, fake, R,
                                            4, b, n, None)
    assert place(C.CSLA_CP_MAX_RANKS + 1, arr(0, 0), arr(1, 1)) == C.CSLA_ERR_ARG
    assert place(2, arr(0, -1), arr(1, 1)) == C.CSLA_ERR_ARG
    assert place(2, arr(0, 4), arr(1, 5)) == C.CSLA_ERR_ARG
    assert place(2, None, arr(1, 1)) == C.CSLA_ERR_ARG
