"""Thin ctypes binding of libcsla (include/csla.h), same entry-point names.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Array arguments may be torch CUDA tensors (their data_ptr is
passed) or raw integer device addresses.  If libcsla.so is missing or cannot
be loaded, importing this module raises: there is no fallback path.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsla.so")

CSLA_OK, CSLA_ERR_ARG, CSLA_ERR_UNSUPPORTED, CSLA_ERR_CUDA, CSLA_ERR_DEVICE = 0, 1, 2, 3, 4
CSLA_F32, CSLA_BF16 = 0, 1
CSLA_VARIANT_AUTO, CSLA_VARIANT_SATURATED, CSLA_VARIANT_STARVED = 0, 1, 2
CSLA_KEY_BF16, CSLA_KEY_E4M3 = 0, 1
CSLA_GATE_TOKEN, CSLA_GATE_CHANNEL = 0, 1
CSLA_OP_INDEXER, CSLA_OP_TOPK, CSLA_OP_CSA_ATTEND, CSLA_OP_HCA_ATTEND, CSLA_OP_CSA_DECODE_STEP = 1, 2, 3, 4, 5
CSLA_OP_INDEXER_TOPK = 6
CSLA_DEVERR_PAGE, CSLA_DEVERR_INDEX, CSLA_DEVERR_LEN, CSLA_DEVERR_TIMEOUT, CSLA_DEVERR_RANGE = 1, 2, 4, 8, 16
CSLA_PAGE_TOKENS = 128

EXPORTS = ("csla_compress_append", "csla_indexer_scores", "csla_topk_select", "csla_csa_attend",
           "csla_hca_attend", "csla_workspace_size", "csla_device_error", "csla_strerror", "csla_version",
           "csla_indexer_scores_noalloc", "csla_window_rows", "csla_csa_decode_step", "csla_check_wait_timeout",
           "csla_cp_record_bytes", "csla_cp_select", "csla_cp_place", "csla_indexer_topk")
CSLA_CP_MAX_RANKS = 64
CSLA_NOALLOC_INDEXER_SCRATCH_BYTES = 786432


class csla_cfg(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int32), ("D", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("H", ctypes.c_int32), ("HI", ctypes.c_int32), ("dI", ctypes.c_int32),
                ("dc", ctypes.c_int32), ("n_win", ctypes.c_int32), ("rope_theta", ctypes.c_float),
                ("eps", ctypes.c_float), ("key_fmt", ctypes.c_int32), ("gate", ctypes.c_int32)]


class csla_cache(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("kidx", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("bt_stride", ctypes.c_int32),
                ("n_pages", ctypes.c_int32), ("kscale", ctypes.c_void_p)]


class csla_state(ctypes.Structure):
    _fields_ = [("win_rows", ctypes.c_void_p), ("win_scales", ctypes.c_void_p),
                ("tail_kv", ctypes.c_void_p), ("tail_idx", ctypes.c_void_p), ("len", ctypes.c_void_p),
                ("n_slots", ctypes.c_int32)]


class csla_compress_params(ctypes.Structure):
    _fields_ = [("gamma_kv", ctypes.c_void_p), ("wg", ctypes.c_void_p), ("gb", ctypes.c_void_p),
                ("wgi", ctypes.c_void_p), ("gbi", ctypes.c_void_p)]


class csla_queries(ctypes.Structure):
    """Query rows other than each request's latest token (see include/csla.h)."""
    _fields_ = [("q_len", ctypes.c_void_p), ("win_rows", ctypes.c_void_p), ("win_scales", ctypes.c_void_p),
                ("win_base", ctypes.c_void_p), ("n_win_rows", ctypes.c_int32), ("one_request", ctypes.c_int32)]


class csla_token_rows(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("stride", ctypes.c_int32),
                ("offset", ctypes.c_int32)]


def queries(q_len, win_rows=None, win_scales=None, win_base=None, n_win_rows=0, one_request=False):
    """csla_queries from tensors (or device addresses); the struct keeps the
    tensors alive for as long as it lives."""
    q = csla_queries(_ptr(q_len), _ptr(win_rows), _ptr(win_scales), _ptr(win_base), int(n_win_rows),
                     1 if one_request else 0)
    q._keep = (q_len, win_rows, win_scales, win_base)
    return q


def token_rows(rows, scales, stride, offset=0):
    """csla_token_rows from tensors (or device addresses), kept alive by the struct."""
    t = csla_token_rows(_ptr(rows), _ptr(scales), int(stride), int(offset))
    t._keep = (rows, scales)
    return t


class CslaError(RuntimeError):
    def __init__(self, fn, status, bits=0):
        self.status, self.bits = status, bits
        super().__init__("%s failed: %s (status %d, device bits 0x%x)"
                         % (fn, _lib.csla_strerror(status).decode(), status, bits))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libcsla.so not built (%s); run `python "
                          "compressed_sparse_long_append_b200/build.py`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "csla_compress_append": [P, P, P, P, I, I, P, P, I, P, P, P],
        "csla_window_rows": [P, P, P, I, I, P, P, I, P],
        "csla_indexer_scores": [P, P, P, P, I, P, I, P, I, P, I, P, P, I, P, Z, P],
        "csla_topk_select": [P, P, P, I, P, I, P, I, I, P, P],
        "csla_indexer_topk": [P, P, P, P, I, P, I, P, I, P, I, P, I, P, P, I, P, Z, P],
        "csla_csa_attend": [P, P, P, P, I, P, P, I, P, I, P, P, P, I, I, P, Z, P],
        "csla_hca_attend": [P, P, P, P, I, P, I, P, I, P, P, P, I, I, P, Z, P],
        "csla_workspace_size": [P, I, I, I],
        "csla_device_error": [P, ctypes.POINTER(ctypes.c_uint32)],
        "csla_strerror": [ctypes.c_int],
        "csla_version": [],
        "csla_check_wait_timeout": [ctypes.c_uint32, P],
        "csla_cp_record_bytes": [P],
        "csla_cp_select": [P, P, P, I, I, I, I, P, P],
        "csla_cp_place": [P, P, P, I, P, I, I, P, P, P],
        "csla_indexer_scores_noalloc": [P, P, P, P, I, P, I, P, I, P, I, P, P, I, P],
        "csla_csa_decode_step": [P, P, P, P, I, I, I, P, P, I, P, P, I, P, I, P, P, I, I, P, P, I, P, P, P, I, I,
                                 P, Z, P, Z, P],
    }
    res = {"csla_workspace_size": ctypes.c_size_t, "csla_strerror": ctypes.c_char_p,
           "csla_cp_record_bytes": ctypes.c_int32}
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res.get(name, ctypes.c_int)
    return L


_lib = _load()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(fn, rc):
    if rc != CSLA_OK:
        raise CslaError(fn, rc)
    return rc


def _ref(s):
    return None if s is None else ctypes.byref(s)


def csla_compress_append(cfg, st, cache, slots, B, T, kv_new, kidx_new, kv_dtype, params, stream=None, tok=None):
    """tok: optional csla_token_rows receiving every new token's window row."""
    return _check("csla_compress_append", _lib.csla_compress_append(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, T, _ptr(kv_new), _ptr(kidx_new), kv_dtype,
        _ref(params), _ref(tok), _stream(stream)))


def csla_window_rows(cfg, st, slots, B, n, rows_out, scales_out, stride, stream=None):
    return _check("csla_window_rows", _lib.csla_window_rows(
        _ref(cfg), _ref(st), _ptr(slots), B, n, _ptr(rows_out), _ptr(scales_out), stride, _stream(stream)))


def csla_indexer_scores(cfg, st, cache, slots, B, max_len, cq, cq_dtype, W_iq, w_dtype, head_w, scores,
                        scores_stride, workspace, workspace_bytes, stream=None, qs=None):
    """qs: optional csla_queries (per-row visible lengths)."""
    return _check("csla_indexer_scores", _lib.csla_indexer_scores(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, _ref(qs), max_len, _ptr(cq), cq_dtype, _ptr(W_iq), w_dtype,
        _ptr(head_w), _ptr(scores), scores_stride, _ptr(workspace), workspace_bytes, _stream(stream)))


def csla_indexer_scores_noalloc(cfg, st, cache, slots, B, max_len, cq, cq_dtype, W_iq, w_dtype, head_w,
                                scores, scores_stride, stream=None, qs=None):
    """The indexer for callers that cannot allocate device memory: same
    inputs and outputs as csla_indexer_scores, no workspace (the library's
    fixed scratch array is used; see include/csla.h for the limit and the
    rule that overlapping calls race)."""
    return _check("csla_indexer_scores_noalloc", _lib.csla_indexer_scores_noalloc(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, _ref(qs), max_len, _ptr(cq), cq_dtype, _ptr(W_iq), w_dtype,
        _ptr(head_w), _ptr(scores), scores_stride, _stream(stream)))


def csla_topk_select(cfg, st, slots, B, max_len, scores, scores_stride, k, idx, stream=None, qs=None):
    return _check("csla_topk_select", _lib.csla_topk_select(
        _ref(cfg), _ref(st), _ptr(slots), B, _ref(qs), max_len, _ptr(scores), scores_stride, k, _ptr(idx),
        _stream(stream)))


def csla_indexer_topk(cfg, st, cache, slots, B, max_len, cq, cq_dtype, W_iq, w_dtype, head_w, k, idx, scores,
                      scores_stride, workspace, workspace_bytes, stream=None, qs=None):
    """csla_indexer_scores + csla_topk_select in one call (same idx); the
    scores of long rows are not stored (`scores` is scratch for rows that
    fall back to the two-step path)."""
    return _check("csla_indexer_topk", _lib.csla_indexer_topk(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, _ref(qs), max_len, _ptr(cq), cq_dtype, _ptr(W_iq), w_dtype,
        _ptr(head_w), k, _ptr(idx), _ptr(scores), scores_stride, _ptr(workspace), workspace_bytes, _stream(stream)))


def csla_csa_attend(cfg, st, cache, slots, B, q, q_dtype, idx, k, sink, gamma_q, out, out_dtype, variant,
                    workspace, workspace_bytes, stream=None, qs=None):
    return _check("csla_csa_attend", _lib.csla_csa_attend(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, _ref(qs), _ptr(q), q_dtype, _ptr(idx), k, _ptr(sink),
        _ptr(gamma_q), _ptr(out), out_dtype, variant, _ptr(workspace), workspace_bytes, _stream(stream)))


def csla_hca_attend(cfg, st, cache, slots, B, max_len, q, q_dtype, sink, gamma_q, out, out_dtype, variant,
                    workspace, workspace_bytes, stream=None, qs=None):
    return _check("csla_hca_attend", _lib.csla_hca_attend(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, _ref(qs), max_len, _ptr(q), q_dtype, _ptr(sink),
        _ptr(gamma_q), _ptr(out), out_dtype, variant, _ptr(workspace), workspace_bytes, _stream(stream)))


def csla_csa_decode_step(cfg, st, cache, slots, B, T, max_len, kv_new, kidx_new, kv_dtype, params, cq, cq_dtype,
                         W_iq, w_dtype, head_w, scores, scores_stride, k, idx, q, q_dtype, sink, gamma_q, out,
                         out_dtype, variant, ws_indexer, ws_indexer_bytes, ws_step, ws_step_bytes, stream=None):
    """compress_append + indexer_scores + topk_select + csa_attend in one call
    (same results; the indexer overlaps the append, see include/csla.h)."""
    return _check("csla_csa_decode_step", _lib.csla_csa_decode_step(
        _ref(cfg), _ref(st), _ref(cache), _ptr(slots), B, T, max_len, _ptr(kv_new), _ptr(kidx_new), kv_dtype,
        _ref(params), _ptr(cq), cq_dtype, _ptr(W_iq), w_dtype, _ptr(head_w), _ptr(scores), scores_stride, k,
        _ptr(idx), _ptr(q), q_dtype, _ptr(sink), _ptr(gamma_q), _ptr(out), out_dtype, variant, _ptr(ws_indexer),
        ws_indexer_bytes, _ptr(ws_step), ws_step_bytes, _stream(stream)))


def csla_workspace_size(cfg, op, B, max_len):
    return int(_lib.csla_workspace_size(_ref(cfg), op, B, max_len))


def indexer_topk_layout(B, HI, dI):
    """Byte offsets of the parts of a csla_indexer_topk workspace, for
    reading its per-row diagnostics after a call: query terms, sample
    scores [B][1024] f32, thresholds [B], candidate counts [B][4] and row
    flags [B] (int32; 1 = the row took the stored-score path), candidates
    [B][4][2048] (key, entry); each part 16-byte aligned.  "total" equals
    csla_workspace_size(cfg, CSLA_OP_INDEXER_TOPK, B, .)."""
    up16 = lambda x: (x + 15) // 16 * 16
    nq = (3 * HI + 15) // 16 * 16
    lay = {"sample": up16(B * nq * dI * 2)}
    lay["t0"] = lay["sample"] + up16(B * 1024 * 4)
    lay["counts"] = lay["t0"] + up16(B * 4)
    lay["flags"] = lay["counts"] + up16(B * 16)
    lay["cand"] = lay["flags"] + up16(B * 4)
    lay["total"] = lay["cand"] + B * 8192 * 8
    return lay


def csla_device_error(stream=None):
    """Synchronise the stream; return (status, bits) of the device error word (cleared)."""
    bits = ctypes.c_uint32(0)
    rc = _lib.csla_device_error(_stream(stream), ctypes.byref(bits))
    return rc, bits.value


def csla_strerror(status):
    return _lib.csla_strerror(status).decode()


def csla_cp_record_bytes(cfg):
    return int(_lib.csla_cp_record_bytes(_ref(cfg)))


def csla_cp_select(cfg, st, cache, slot, b_lo, n, E_max, recs, stream=None):
    return _check("csla_cp_select", _lib.csla_cp_select(_ref(cfg), _ref(st), _ref(cache), slot, b_lo, n, E_max,
                                                        _ptr(recs), _stream(stream)))


def csla_cp_place(cfg, st, cache, slot, recs, E_max, b_lo, n, stream=None):
    """b_lo, n: sequences of R ints (host)."""
    R = len(b_lo)
    arr = ctypes.c_int32 * max(R, 1)
    return _check("csla_cp_place", _lib.csla_cp_place(_ref(cfg), _ref(st), _ref(cache), slot, _ptr(recs), R,
                                                      E_max, arr(*b_lo), arr(*n), _stream(stream)))


def csla_check_wait_timeout(limit_us, stream=None):
    return _check("csla_check_wait_timeout", _lib.csla_check_wait_timeout(int(limit_us), _stream(stream)))


def csla_version():
    return int(_lib.csla_version())
