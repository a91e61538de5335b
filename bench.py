#!/usr/bin/env python
"""Decode-step benchmark of the CSA/HCA compressed-attention path on B200.

One step = one decode token for every request of a CSA layer:
  csla_compress_append (T=1) -> csla_indexer_scores -> csla_topk_select ->
  csla_csa_attend.
Workload (default): 8 requests at 131072-token context, m=4 (32768
compressed entries each), 64 query heads, head_dim 512 (448 fp8 + 64 bf16
RoPE dims), dc=1024 -> 16 index heads of 128, top-k 512, window 128.
An HCA layer (4 requests at 1,048,576 tokens, m'=128) is measured after it
and reported in the same JSON line under "hca_decode", then a CSA prefill
chunk (4096 new tokens and their queries after a 262144-token prefix, top-k
1024; indexer and top-k as one csla_indexer_topk call) under "csa_prefill".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N>1 runs under torchrun: every rank serves its own 8 requests (weak scaling,
no collective on the data path); the step time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA decode tokens/s and achieved HBM GB/s vs roofline, 1×B200"
UNIT = "tokens/s"
CSA = dict(B=8, L=131072, m=4, H=64, D=512, HI=16, dI=128, dc=1024, k=512, n_win=128)
HCA = dict(B=4, L=1048576, m=128, H=64, D=512, n_win=128)
CHUNK = 16384          # tokens per compress call while building the caches
CSA_COPIES = 4         # layer copies rotated per step: 4 x ~75 MB touched > 2 x L2
HCA_COPIES = 14        # 14 x ~19.3 MB
HEADROOM = 256         # cache capacity beyond the nominal context (tokens appended while timing)
PREFILL = dict(T=4096, L0=262144, m=4, H=64, D=512, HI=16, dI=128, dc=1024, k=1024, n_win=128)
NW = 127               # window rows from before a prefill chunk that its first query needs


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-hca", action="store_true", help="skip the HCA layer measurement")
    ap.add_argument("--no-prefill", action="store_true", help="skip the CSA prefill-chunk measurement")
    ap.add_argument("--prefill-only", action="store_true", help="only the CSA prefill-chunk measurement")
    ap.add_argument("--no-e4m3", action="store_true", help="skip the CSA decode leg with E4M3 index keys")
    ap.add_argument("--hca-only", action="store_true", help="only the HCA decode measurement")
    ap.add_argument("--e4m3-only", action="store_true", help="only the CSA decode leg with E4M3 index keys")
    ap.add_argument("--no-invariance", action="store_true",
                    help="skip the ragged 64-request CSA + HCA decode measurement")
    ap.add_argument("--no-stack", action="store_true",
                    help="skip the interleaved CSA/HCA layer stack on one shared block table")
    ap.add_argument("--stack-layers", type=int, default=8, help="layers of the interleaved stack")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", type=int, default=0, help="attention variant: 0 auto, 1 saturated, 2 starved")
    ap.add_argument("--fused-step", action="store_true",
                    help="time the CSA step as csla_csa_decode_step instead of the four separate library calls")
    ap.add_argument("--profile", action="store_true",
                    help="only the timed steps of the first leg run (CSA decode; the prefill chunk with "
                         "--prefill-only; the HCA step with --hca-only; the E4M3-key CSA step with --e4m3-only), "
                         "bracketed by cudaProfilerStart/Stop (for ncu --profile-from-start off); implies "
                         "--no-hca --no-cpu-baseline and no e2e leg")
    return ap.parse_args()


def tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops_sustained"]), "measured (sustained)"
    except Exception:
        return 1400.0, "fallback (sustained)"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if len(r) > 2 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) > 2 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            for i, n in enumerate(names):
                if len(r) > 5 + i and r[5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workload build
def build_layer(shape_kw, n_req, L0s, seed, rank, device, block_table=None):
    """Caches of n_req requests after appending L0s[r] tokens to request r,
    through csla_compress_append on raw streams generated on the device.
    block_table: a filled table shared with other layers (else the layer's
    own, a seeded page permutation)."""
    import torch
    from compressed_sparse_long_append_b200 import csla as C
    from compressed_sparse_long_append_b200.layer import CompressParams, LayerBuffers, LayerShape
    from csla_synth import permutation, normal
    from csla_synth import torch_gen

    sh = LayerShape(m=shape_kw["m"], D=shape_kw["D"], H=shape_kw["H"], HI=shape_kw.get("HI", 16),
                    dI=shape_kw.get("dI", 128), dc=shape_kw.get("dc", 1024), n_win=shape_kw["n_win"],
                    key_fmt=shape_kw.get("key_fmt", 0))
    L_cap = shape_kw["L"] + HEADROOM
    pages_per = -(-L_cap // 128)
    n_pages = n_req * pages_per
    lb = LayerBuffers(sh, n_req, n_pages, pages_per, device, block_table=block_table)
    if block_table is None:
        perm = permutation(seed, "pages/%d" % rank, n_pages).astype("int32").reshape(n_req, pages_per)
        lb.block_table.copy_(torch.from_numpy(perm))
    D, dI, m = sh.D, sh.dI, sh.m
    g = lambda name, shp, std=1.0: torch.as_tensor(normal(seed, name, shp, std=std), dtype=torch.float32)
    cp = CompressParams(1.0 + 0.1 * g("gamma_kv", (D,)), g("wg", (D,), 1.0 / D ** 0.5), g("gb", (m,)),
                        g("wgi", (dI,), 1.0 / dI ** 0.5) if sh.is_csa else None,
                        g("gbi", (m,)) if sh.is_csa else None, device)
    for r in range(n_req):
        slots = torch.tensor([r], dtype=torch.int32, device=device)
        for a in range(0, L0s[r], CHUNK):
            b = min(L0s[r], a + CHUNK)
            kv = torch_gen.normal(seed, "kv/%d/%d" % (rank, r), (b - a, D), start=a * D, device=device) \
                .to(torch.bfloat16)
            ki = torch_gen.normal(seed, "idx/%d/%d" % (rank, r), (b - a, dI), start=a * dI, device=device) \
                .to(torch.bfloat16) if sh.is_csa else None
            C.csla_compress_append(lb.cfg(), lb.state(), lb.cache(), slots, 1, b - a, kv, ki, C.CSLA_BF16,
                                   cp.struct())
    torch.cuda.synchronize()
    params = {"sink": g("sink", (sh.H,)).to(device), "gamma_q": (1.0 + 0.1 * g("gamma_q", (D,))).to(device)}
    if sh.is_csa:
        params["W_iq"] = torch_gen.normal(seed, "W_iq", (sh.HI * dI, sh.dc), device=device,
                                          std=1.0 / sh.dc ** 0.5).to(torch.bfloat16)
    return lb, cp, params


def step_inputs(shape_kw, n_req, n_steps, seed, rank, device):
    """Per-step inputs for all steps, device-resident, plus pinned host copies."""
    import torch
    from csla_synth import torch_gen
    B, H, D = n_req, shape_kw["H"], shape_kw["D"]
    out = []
    for s in range(n_steps):
        d = {"q": torch_gen.normal(seed, "q/%d/%d" % (rank, s), (B, H, D), device=device).to(torch.bfloat16),
             "kv": torch_gen.normal(seed, "kvn/%d/%d" % (rank, s), (B, 1, D), device=device).to(torch.bfloat16)}
        if shape_kw["m"] == 4:
            d["kidx"] = torch_gen.normal(seed, "kin/%d/%d" % (rank, s), (B, 1, shape_kw["dI"]),
                                         device=device).to(torch.bfloat16)
            d["cq"] = torch_gen.normal(seed, "cq/%d/%d" % (rank, s), (B, shape_kw["dc"]), device=device) \
                .to(torch.bfloat16)
            d["head_w"] = torch_gen.normal(seed, "hw/%d/%d" % (rank, s), (B, shape_kw["HI"]), device=device) \
                .to(torch.float32)
        d["host"] = {k: v.cpu().pin_memory() for k, v in d.items()}
        out.append(d)
    return out


class CsaStep:
    """One CSA decode step of one layer copy: csla_csa_decode_step (or, with
    fused=False, the four separate library calls); each call takes the step's
    input tensors x (dict of device tensors).  sep_calls are the four
    separate calls (per-call timings, the indexer roofline)."""

    fused = False

    def __init__(self, lb, cp, params, kw, variant, device):
        import torch
        from compressed_sparse_long_append_b200 import csla as C
        self.C, self.lb, self.cp, self.p, self.kw, self.variant = C, lb, cp, params, kw, variant
        B = kw["B"]
        self.B = B
        self.slots = torch.arange(B, dtype=torch.int32, device=device)
        self.max_len = kw["L"] + HEADROOM
        self.stride = self.max_len // kw["m"]
        self.scores = torch.zeros((B, self.stride), dtype=torch.float32, device=device)
        self.idx = torch.zeros((B, kw["k"]), dtype=torch.int32, device=device)
        self.out = torch.zeros((B, kw["H"], kw["D"]), dtype=torch.bfloat16, device=device)
        cfg = lb.cfg()
        self.wsi = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER, B, self.max_len)
        self.wsa = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, B, kw["k"])
        self.ws_i = torch.zeros(self.wsi, dtype=torch.uint8, device=device)
        self.ws_a = torch.zeros(self.wsa, dtype=torch.uint8, device=device)
        self.wss = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_DECODE_STEP, B, kw["k"])
        self.ws_s = torch.zeros(self.wss, dtype=torch.uint8, device=device)
        self.cfg, self.st, self.cache, self.cps = cfg, lb.state(), lb.cache(), cp.struct()
        self.names = ["compress_append", "indexer_scores", "topk_select", "csa_attend"]
        self.sep_calls = [self._compress, self._indexer, self._topk, self._attend]
        self.calls = [self._step] if self.fused else self.sep_calls

    def _step(self, x):
        C = self.C
        C.csla_csa_decode_step(self.cfg, self.st, self.cache, self.slots, self.B, 1, self.max_len, x["kv"],
                               x["kidx"], C.CSLA_BF16, self.cps, x["cq"], C.CSLA_BF16, self.p["W_iq"], C.CSLA_BF16,
                               x["head_w"], self.scores, self.stride, self.kw["k"], self.idx, x["q"], C.CSLA_BF16,
                               self.p["sink"], self.p["gamma_q"], self.out, C.CSLA_BF16, self.variant, self.ws_i,
                               self.wsi, self.ws_s, self.wss)

    def _compress(self, x):
        C = self.C
        C.csla_compress_append(self.cfg, self.st, self.cache, self.slots, self.B, 1, x["kv"], x["kidx"],
                               C.CSLA_BF16, self.cps)

    def _indexer(self, x):
        C = self.C
        C.csla_indexer_scores(self.cfg, self.st, self.cache, self.slots, self.B, self.max_len, x["cq"],
                              C.CSLA_BF16, self.p["W_iq"], C.CSLA_BF16, x["head_w"], self.scores, self.stride,
                              self.ws_i, self.wsi)

    def _topk(self, x):
        self.C.csla_topk_select(self.cfg, self.st, self.slots, self.B, self.max_len, self.scores, self.stride,
                                self.kw["k"], self.idx)

    def _attend(self, x):
        C = self.C
        C.csla_csa_attend(self.cfg, self.st, self.cache, self.slots, self.B, x["q"], C.CSLA_BF16, self.idx,
                          self.kw["k"], self.p["sink"], self.p["gamma_q"], self.out, C.CSLA_BF16, self.variant,
                          self.ws_a, self.wsa)

    def launches(self):
        return csa_launches(self.kw, self.variant, self.fused)


def csa_launches(kw, variant, fused):
    """Kernels of one CSA step: compress (pool + tail/len), iq_project +
    indexer, topk, attend, + combine unless the saturated variant runs
    (forced, or automatic: one chunk per request or B >= SM count); the
    fused step adds the length snapshot and the second indexer launch."""
    return 2 + 2 + 1 + attend_launches(kw["k"] + kw["n_win"], kw["B"], variant) + (2 if fused else 0)


def attend_launches(rows, B, variant):
    """Attention kernels of one call over `rows` rows per request: the
    attention, plus the combine unless the saturated variant runs."""
    # the library's bound on a call's chunk count (the starved grid's width)
    max_chunks = min(32, max(1, -(-rows // 64)))
    saturated = variant == 1 or (variant == 0 and (B >= 148 or max_chunks <= 1))
    return 1 + (0 if saturated else 1)


class HcaStep:
    """One HCA decode step: compress_append then hca_attend."""

    def __init__(self, lb, cp, params, kw, variant, device):
        import torch
        from compressed_sparse_long_append_b200 import csla as C
        self.C, self.lb, self.cp, self.p, self.kw, self.variant = C, lb, cp, params, kw, variant
        B = kw["B"]
        self.B = B
        self.slots = torch.arange(B, dtype=torch.int32, device=device)
        self.max_len = kw["L"] + HEADROOM
        self.out = torch.zeros((B, kw["H"], kw["D"]), dtype=torch.bfloat16, device=device)
        cfg = lb.cfg()
        self.wsa = C.csla_workspace_size(cfg, C.CSLA_OP_HCA_ATTEND, B, self.max_len)
        self.ws_a = torch.zeros(self.wsa, dtype=torch.uint8, device=device)
        self.cfg, self.st, self.cache, self.cps = cfg, lb.state(), lb.cache(), cp.struct()
        self.names = ["compress_append", "hca_attend"]
        self.calls = [self._compress, self._attend]
        self.sep_calls = self.calls

    def _compress(self, x):
        C = self.C
        C.csla_compress_append(self.cfg, self.st, self.cache, self.slots, self.B, 1, x["kv"], None,
                               C.CSLA_BF16, self.cps)

    def _attend(self, x):
        C = self.C
        C.csla_hca_attend(self.cfg, self.st, self.cache, self.slots, self.B, self.max_len, x["q"], C.CSLA_BF16,
                          self.p["sink"], self.p["gamma_q"], self.out, C.CSLA_BF16, self.variant, self.ws_a,
                          self.wsa)


class PrefillStep:
    """One CSA prefill chunk of one request: the ring snapshot of the NW
    positions before the chunk, the chunk's append (T tokens, every token's
    window row kept), then the T queries (query i at position L0+i) through
    the indexer and top-k (one csla_indexer_topk call: the rows' scores are
    not stored) and attention with per-row visible lengths and the window
    rows from the chunk buffer.  A last pair of device copies puts the
    request's length and ring back to their pre-chunk state, so that every
    step does the same work (the appended entries are rewritten with the same
    bytes)."""

    def __init__(self, lb, cp, params, kw, variant, device):
        import torch
        from compressed_sparse_long_append_b200 import csla as C
        self.C, self.lb, self.cp, self.p, self.kw, self.variant = C, lb, cp, params, kw, variant
        T, L0, k = kw["T"], kw["L0"], kw["k"]
        L1 = L0 + T
        self.T, self.max_len, self.stride = T, L1, L1 // kw["m"]
        rb = (kw["D"] - 64) + 2 * 64
        self.slot = torch.zeros(1, dtype=torch.int32, device=device)
        self.rows_slots = torch.zeros(T, dtype=torch.int32, device=device)
        self.buf = torch.zeros((NW + T, rb), dtype=torch.uint8, device=device)
        self.bufsc = torch.zeros(NW + T, dtype=torch.float32, device=device)
        self.q_len = torch.arange(L0 + 1, L1 + 1, dtype=torch.int32, device=device)
        self.base = torch.full((T,), NW - L0, dtype=torch.int32, device=device)
        self.qs_rows = C.queries(self.q_len, one_request=True)
        self.qs_att = C.queries(self.q_len, self.buf, self.bufsc, self.base, NW + T)
        self.tok = C.token_rows(self.buf, self.bufsc, NW + T, NW)
        self.scores = torch.zeros((T, self.stride), dtype=torch.float32, device=device)
        self.idx = torch.zeros((T, k), dtype=torch.int32, device=device)
        self.out = torch.zeros((T, kw["H"], kw["D"]), dtype=torch.bfloat16, device=device)
        cfg = lb.cfg()
        self.wsi = C.csla_workspace_size(cfg, C.CSLA_OP_INDEXER_TOPK, T, self.max_len)
        self.wsa = C.csla_workspace_size(cfg, C.CSLA_OP_CSA_ATTEND, T, k)
        self.ws_i = torch.zeros(self.wsi, dtype=torch.uint8, device=device)
        self.ws_a = torch.zeros(self.wsa, dtype=torch.uint8, device=device)
        self.len0, self.win0, self.wsc0 = lb.len.clone(), lb.win_rows.clone(), lb.win_scales.clone()
        self.cfg, self.st, self.cache, self.cps = cfg, lb.state(), lb.cache(), cp.struct()
        self.names = ["window_rows", "compress_append", "indexer_topk", "csa_attend", "rewind"]
        self.calls = [self._snapshot, self._compress, self._indexer_topk, self._attend, self._rewind]
        # the same selection as two calls (scores stored, then read), timed beside it
        self.two_call_names = ["indexer_scores", "topk_select"]
        self.two_calls = [self._indexer, self._topk]

    def selection_stats(self):
        """Rows that fell back to stored scores, and the candidate counts of
        the others (read from the csla_indexer_topk workspace: query terms,
        sample scores, thresholds, four counts per row, flags)."""
        import numpy as np
        import torch
        T, kw = self.T, self.kw
        lay = self.C.indexer_topk_layout(T, kw["HI"], kw["dI"])
        o_cnt, o_flag = lay["counts"], lay["flags"]
        cnt = self.ws_i[o_cnt:o_cnt + 16 * T].view(torch.int32).cpu().numpy().reshape(T, 4).sum(axis=1)
        flag = self.ws_i[o_flag:o_flag + 4 * T].view(torch.int32).cpu().numpy()
        ok = flag == 0
        return int((~ok).sum()), float(np.mean(cnt[ok])) if ok.any() else 0.0, int(cnt.max())

    def _snapshot(self, x):
        self.C.csla_window_rows(self.cfg, self.st, self.slot, 1, NW, self.buf, self.bufsc, NW + self.T)

    def _compress(self, x):
        C = self.C
        C.csla_compress_append(self.cfg, self.st, self.cache, self.slot, 1, self.T, x["kv"], x["kidx"],
                               C.CSLA_BF16, self.cps, tok=self.tok)

    def _indexer(self, x):
        C = self.C
        C.csla_indexer_scores(self.cfg, self.st, self.cache, self.rows_slots, self.T, self.max_len, x["cq"],
                              C.CSLA_BF16, self.p["W_iq"], C.CSLA_BF16, x["head_w"], self.scores, self.stride,
                              self.ws_i, self.wsi, qs=self.qs_rows)

    def _indexer_topk(self, x):
        C = self.C
        C.csla_indexer_topk(self.cfg, self.st, self.cache, self.rows_slots, self.T, self.max_len, x["cq"],
                            C.CSLA_BF16, self.p["W_iq"], C.CSLA_BF16, x["head_w"], self.kw["k"], self.idx,
                            self.scores, self.stride, self.ws_i, self.wsi, qs=self.qs_rows)

    def _topk(self, x):
        self.C.csla_topk_select(self.cfg, self.st, self.rows_slots, self.T, self.max_len, self.scores, self.stride,
                                self.kw["k"], self.idx, qs=self.qs_rows)

    def _attend(self, x):
        C = self.C
        C.csla_csa_attend(self.cfg, self.st, self.cache, self.rows_slots, self.T, x["q"], C.CSLA_BF16, self.idx,
                          self.kw["k"], self.p["sink"], self.p["gamma_q"], self.out, C.CSLA_BF16, self.variant,
                          self.ws_a, self.wsa, qs=self.qs_att)

    def _rewind(self, x):
        self.lb.len.copy_(self.len0)
        self.lb.win_rows.copy_(self.win0)
        self.lb.win_scales.copy_(self.wsc0)

    def flops(self):
        """Algorithmic tensor FLOPs of the chunk's queries: indexer
        2*HI*dI per visible entry per query; attention 4*H*D per set row
        (q.k and p.v) per query."""
        kw = self.kw
        L = [kw["L0"] + 1 + i for i in range(self.T)]
        fi = sum(2 * kw["HI"] * kw["dI"] * (x // kw["m"]) for x in L)
        fa = sum(4 * kw["H"] * kw["D"] * (min(kw["k"], x // kw["m"]) + min(kw["n_win"], x)) for x in L)
        return fi, fa


def prefill_leg(W, K, seed, rank, world, device, variant, profile=False):
    """Times the prefill chunk: one CUDA graph of the whole step (five library
    calls and the rewind copies) replayed K times between one event pair."""
    import torch
    from csla_synth import torch_gen
    kw = dict(PREFILL)
    T, L0 = kw["T"], kw["L0"]
    lb, cp, params = build_layer(dict(kw, B=1, L=L0 + T), 1, [L0], seed, rank, device)
    x = {"q": torch_gen.normal(seed, "pq/%d" % rank, (T, kw["H"], kw["D"]), device=device).to(torch.bfloat16),
         "kv": torch_gen.normal(seed, "kv/%d/0" % rank, (T, kw["D"]), start=L0 * kw["D"], device=device)
         .to(torch.bfloat16),
         "kidx": torch_gen.normal(seed, "idx/%d/0" % rank, (T, kw["dI"]), start=L0 * kw["dI"], device=device)
         .to(torch.bfloat16),
         "cq": torch_gen.normal(seed, "pcq/%d" % rank, (T, kw["dc"]), device=device).to(torch.bfloat16),
         "head_w": torch_gen.normal(seed, "phw/%d" % rank, (T, kw["HI"]), device=device).to(torch.float32)}
    st = PrefillStep(lb, cp, params, kw, variant, device)
    for _ in range(W):
        for c in st.calls:
            c(x)
    torch.cuda.synchronize()
    g = capture(lambda: [c(x) for c in st.calls])
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if profile:
        torch.cuda.profiler.start()
    e0.record()
    for _ in range(K):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    if profile:
        torch.cuda.profiler.stop()
    ms = dp_max(e0.elapsed_time(e1) / K, world, device)
    del g
    fb_rows, cand_mean, cand_max = st.selection_stats()
    # per-call times: each call its own graph, one event pair around each
    # replay; the two-call selection, for comparison, right after the fused
    # call (before the rewind, which leaves the queries past the length)
    order = st.calls[:3] + st.two_calls + st.calls[3:]
    order_names = st.names[:3] + st.two_call_names + st.names[3:]
    gs = [capture(lambda c=c: c(x)) for c in order]
    seg = [0.0] * len(gs)
    for _ in range(max(1, K // 2)):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(gs) + 1)]
        ev[0].record()
        for j, gg in enumerate(gs):
            gg.replay()
            ev[j + 1].record()
        torch.cuda.synchronize()
        for j in range(len(gs)):
            seg[j] += ev[j].elapsed_time(ev[j + 1]) / max(1, K // 2)
    del gs
    fi, fa = st.flops()
    tpk, tkind = tensor_peak()
    tf = (fi + fa) / (ms * 1e-3) / 1e12
    sg = dict(zip(order_names, seg))
    out = {"workload": "csa_prefill_T4096_L262144", "tokens_per_s": T * world / (ms * 1e-3), "ms_per_chunk": ms,
           "queries": T, "prefix": L0, "topk": kw["k"],
           "segments_ms": {n: sg[n] for n in st.names},
           "two_call_selection_ms": {n: sg[n] for n in st.two_call_names},
           "selection": {"fallback_rows": fb_rows, "mean_candidates": cand_mean, "max_candidates": cand_max},
           "algorithmic_tflop": (fi + fa) / 1e12, "indexer_tflop": fi / 1e12, "attend_tflop": fa / 1e12,
           "tensor_tflops": tf, "tensor_peak": tpk, "tensor_peak_kind": tkind, "tensor_frac": tf / tpk,
           "indexer_topk_tensor_frac": fi / (sg["indexer_topk"] * 1e-3) / 1e12 / tpk,
           "attend_tensor_frac": fa / (sg["csa_attend"] * 1e-3) / 1e12 / tpk,
           "l2": "inputs larger than L2 (q 268 MB; the rows' scores are not stored)",
           "launch": "one CUDA graph per chunk, K replays between one event pair"}
    del st, lb
    torch.cuda.empty_cache()
    return out


def hca_leg(W, K, seed, rank, world, device, variant, peak, profile=False):
    """The HCA layer decode step: 4 requests at 2^20 tokens."""
    import torch
    hk = dict(HCA)
    HR, hm, hB = HCA_COPIES, hk["m"], hk["B"]
    # requests staggered 16 tokens apart inside one block, clear of its end:
    # with fewer than ~78 appends per copy no block closes during the run
    # (in steady decode one closes every 128 steps per request)
    hL0s = [hk["L"] - 127 + 16 * b for b in range(hB)]
    closes = sum(1 for i in range(W, W + K) for b in range(hB) if (hL0s[b] + i // HR + 1) % hm == 0)
    hlb, hcp, hparams = build_layer(hk, hB, hL0s, seed, rank, device)
    hin = step_inputs(hk, hB, W + K, seed, rank, device)
    hsteps = make_copies(HcaStep, hlb, hcp, hparams, hk, variant, device, HR)
    hms = dp_max(run_steps(hsteps, hin, W, K, profile=profile), world, device)
    out = {"workload": "hca_decode_B4_L1048576", "tokens_per_s": hB * world / (hms * 1e-3), "ms_per_step": hms,
           "block_closes_in_timed_steps": closes}
    if not profile:
        hms_att = dp_max(call_time(hsteps, hin, W, K, 1), world, device)
        rows = sum(int(x) // hm for x in hsteps[0].lb.len.tolist()) / hB + hk["n_win"]
        hbytes = hB * (rows * (hk["D"] + 64 + 4) + 2 * hk["H"] * hk["D"] * 2)
        hflops = hB * rows * hk["H"] * hk["D"] * 4
        out.update({"attend_ms": hms_att, "attend_hbm_gbs": hbytes / (hms_att * 1e-3) / 1e9,
                    "attend_hbm_frac": hbytes / (hms_att * 1e-3) / 1e9 / peak,
                    "attend_tflops": hflops / (hms_att * 1e-3) / 1e12,
                    "attend_tensor_frac_sustained": hflops / (hms_att * 1e-3) / 1e12 / 1395.7})
        out["block_close"] = hca_block_close(K, seed, rank, world, device, hk, hcp)
    del hsteps, hlb, hin
    torch.cuda.empty_cache()
    return out


def hca_block_close(K, seed, rank, world, device, hk, hcp):
    """What closing a 128-token HCA block adds to a step: the append of one
    token to 4 requests whose next token closes a block (the block is pooled
    from its 128 raw rows, normed, rotated and quantised) against one whose
    next token does not, each replayed K times with the length put back
    after every append.  One request closes a block every 128 steps, so the
    amortised cost per step is the difference / 128."""
    import torch
    from compressed_sparse_long_append_b200 import csla as C
    from compressed_sparse_long_append_b200.layer import LayerBuffers, LayerShape
    from csla_synth import torch_gen
    B = hk["B"]
    res = {}
    for name, L0 in (("close", 1023), ("open", 1024)):
        kw = dict(hk, B=B, L=2048)
        lb, _, _ = build_layer(kw, B, [L0] * B, seed + 7, rank, device)
        kv = torch_gen.normal(seed + 7, "bc/%d" % rank, (B, 1, hk["D"]), device=device).to(torch.bfloat16)
        slots = torch.arange(B, dtype=torch.int32, device=device)
        len0 = lb.len.clone()
        cfg, st, cache, cps = lb.cfg(), lb.state(), lb.cache(), hcp.struct()

        def step():
            C.csla_compress_append(cfg, st, cache, slots, B, 1, kv, None, C.CSLA_BF16, cps)
            lb.len.copy_(len0)
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        g = capture(lambda: [step() for _ in range(K)])
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        res[name] = dp_max(e0.elapsed_time(e1) / K, world, device) * 1e3
        del g, lb
    extra = res["close"] - res["open"]
    return {"append_us_all_4_close": res["close"], "append_us_none_close": res["open"],
            "extra_us_when_all_close": extra, "amortised_us_per_step": extra / 128,
            "note": "each request closes one block per 128 steps"}


def e4m3_leg(W, K, seed, rank, world, device, variant, profile=False):
    """The headline CSA decode workload (8 x 131072, top-k 512) with its index
    keys stored as E4M3 codes plus one power-of-two scale per entry (132
    instead of 256 bytes per entry): the same step, timed the same way, and
    the indexer call's achieved bandwidth on its algorithmic bytes."""
    import torch
    kw = dict(CSA, key_fmt=1)
    R, m, B = CSA_COPIES, kw["m"], kw["B"]
    before = -(-(W + K) // R)
    L0s = [kw["L"] - before - (b % m) for b in range(B)]
    lb, cp, params = build_layer(kw, B, L0s, seed, rank, device)
    inputs = step_inputs(kw, B, W + K, seed, rank, device)
    CsaStep.fused = False
    steps = make_copies(CsaStep, lb, cp, params, kw, variant, device, R)
    torch.cuda.synchronize()
    ms = dp_max(run_steps(steps, inputs, W, K, profile=profile), world, device)
    if profile:
        return {"workload": "csa_decode_B8_L131072_e4m3_keys", "tokens_per_s": B * world / (ms * 1e-3),
                "ms_per_step": ms}
    seg = breakdown(steps, inputs, W, K)
    ms_idx = call_time(steps, inputs, W, K, 1)
    nv = sum(int(x) // m for st in steps for x in st.lb.len.tolist()) / R
    idx_bytes = nv * (kw["dI"] + 4 + 4) + kw["HI"] * kw["dI"] * kw["dc"] * 2
    peak, peak_kind = peaks()
    achieved = idx_bytes / (ms_idx * 1e-3) / 1e9
    out = {"workload": "csa_decode_B8_L131072_e4m3_keys", "tokens_per_s": B * world / (ms * 1e-3),
           "ms_per_step": ms, "key_bytes_per_entry": kw["dI"] + 4,
           "segments_ms": {"compress_append": seg[0], "indexer_scores": seg[1], "topk_select": seg[2],
                           "csa_attend": seg[3]},
           "indexer": {"call_ms": ms_idx, "algorithmic_bytes": idx_bytes, "achieved_gbs": achieved,
                       "frac": achieved / peak, "peak": peak, "peak_kind": peak_kind,
                       "traffic": indexer_traffic("csla_indexer_scores_e4m3")}}
    del steps, lb, inputs
    torch.cuda.empty_cache()
    return out


def invariance_leg(W, K, seed, rank, world, device, variant):
    """The batch-invariance workload as a throughput number: 64 requests
    with contexts log-uniform in [1K, 1M] tokens (the lengths of the
    invariance test), one decode step = a CSA layer step (top-k 512) and an
    HCA layer step for all 64 requests, one CUDA graph per step.  Caches are
    built by csla_compress_append; they are GBs, far larger than L2."""
    import math
    import torch
    from csla_synth import uniform
    u = uniform(5, "invariance/len", (64,))
    lens = [int(math.exp(math.log(1024) + x * math.log(1024))) for x in u]
    B = len(lens)
    before = W + K
    L0s = [L - before for L in lens]
    ck = dict(CSA, B=B, L=max(lens))
    hk = dict(HCA, B=B, L=max(lens))
    clb, ccp, cpar = build_layer(ck, B, L0s, seed, rank, device)
    hlb, hcp, hpar = build_layer(hk, B, L0s, seed + 1, rank, device)
    cin = step_inputs(ck, B, W + K, seed, rank, device)
    hin = step_inputs(hk, B, W + K, seed + 1, rank, device)
    cs = CsaStep(clb, ccp, cpar, ck, variant, device)
    hs = HcaStep(hlb, hcp, hpar, hk, variant, device)
    for i in range(W):
        for c in cs.calls:
            c(cin[i])
        for c in hs.calls:
            c(hin[i])
    torch.cuda.synchronize()
    graphs = []
    for i in range(W, W + K):
        graphs.append(capture(lambda: ([c(cin[i]) for c in cs.calls], [c(hin[i]) for c in hs.calls])))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for g in graphs:
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = dp_max(e0.elapsed_time(e1) / K, world, device)
    del graphs
    out = {"workload": "invariance_64req_L1K-1M_csa_hca", "tokens_per_s": B * world / (ms * 1e-3),
           "ms_per_step": ms, "requests_per_gpu": B, "context_tokens": sum(lens), "context_min": min(lens),
           "context_max": max(lens), "step": "one CSA layer (top-k 512) + one HCA layer, all requests",
           "l2": "inputs larger than L2 (CSA index keys alone ~600 MB per step)"}
    del cs, hs, clb, hlb, cin, hin
    torch.cuda.empty_cache()
    return out


def stack_leg(W, K, seed, rank, world, device, variant, n_layers):
    """A model-shaped stack: n_layers attention layers, CSA and HCA
    interleaved (CSA first), the headline decode batch (8 requests at 131072
    tokens) going through every layer, all layers paged through ONE block
    table.  One decode step = every layer's step for every request (CSA:
    the four library calls; HCA: append + attend), one CUDA graph per step.
    The layers are independent copies of one built CSA and one built HCA
    layer (the same bytes, separate memory), so the stack touches n_layers
    layers' caches per step, far more than L2."""
    import torch
    from csla_synth import permutation
    kc = dict(CSA)
    kh = dict(HCA, B=kc["B"], L=kc["L"])
    B, m = kc["B"], kc["m"]
    L0s = [kc["L"] - (W + K) - (b % m) for b in range(B)]
    pages_per = -(-(kc["L"] + HEADROOM) // 128)
    bt = torch.from_numpy(permutation(seed, "stack_pages/%d" % rank, B * pages_per).astype("int32")
                          .reshape(B, pages_per)).to(device)
    clb, ccp, cpar = build_layer(kc, B, L0s, seed, rank, device, block_table=bt)
    hlb, hcp, hpar = build_layer(kh, B, L0s, seed + 1, rank, device, block_table=bt)
    cin = step_inputs(kc, B, W + K, seed, rank, device)
    hin = step_inputs(kh, B, W + K, seed + 1, rank, device)
    CsaStep.fused = False
    layers = []
    for i in range(n_layers):
        csa = i % 2 == 0
        base, cp, par = (clb, ccp, cpar) if csa else (hlb, hcp, hpar)
        nb, np_ = (base, par) if i < 2 else clone_layer(base, par, share_block_table=True)
        layers.append((CsaStep if csa else HcaStep)(nb, cp, np_, kc if csa else kh, variant, device))
    assert all(st.lb.block_table.data_ptr() == bt.data_ptr() for st in layers)
    ins = lambda i, j: cin[j] if i % 2 == 0 else hin[j]
    for j in range(W):
        for i, st in enumerate(layers):
            for c in st.calls:
                c(ins(i, j))
    torch.cuda.synchronize()
    graphs = []
    for j in range(W, W + K):
        graphs.append(capture(lambda: [c(ins(i, j)) for i, st in enumerate(layers) for c in st.calls]))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for g in graphs:
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = dp_max(e0.elapsed_time(e1) / K, world, device)
    del graphs
    n_csa = (n_layers + 1) // 2
    hca_launches = 2 + attend_launches(kh["L"] // kh["m"] + kh["n_win"], B, variant)
    launches = n_csa * csa_launches(kc, variant, False) + (n_layers - n_csa) * hca_launches
    out = {"workload": "stack%d_csa_hca_B8_L131072" % n_layers, "layers": n_layers,
           "layer_order": "CSA, HCA, CSA, ... (interleaved)", "tokens_per_s": B * world / (ms * 1e-3),
           "ms_per_step": ms, "us_per_layer": ms * 1e3 / n_layers, "launches_per_step": launches,
           "block_table": "one [8, %d] int32 table shared by all layers" % pages_per,
           "l2": "inputs larger than L2 (%d layers' caches touched per step)" % n_layers}
    del layers, clb, hlb, cin, hin
    torch.cuda.empty_cache()
    return out


def clone_layer(lb, params, share_block_table=False):
    """An independent copy of a layer's device buffers and weights (the
    rotation below walks several such copies, like the layers of a model)."""
    from compressed_sparse_long_append_b200.layer import LayerBuffers
    nb = object.__new__(LayerBuffers)
    nb.__dict__.update(lb.__dict__)
    for k in ("rows", "scales", "kidx", "kscale", "block_table", "win_rows", "win_scales", "tail_kv", "tail_idx",
              "len"):
        if k == "block_table" and share_block_table:
            continue
        v = getattr(lb, k)
        setattr(nb, k, None if v is None else v.clone())
    return nb, {k: v.clone() for k, v in params.items()}


def make_copies(step_cls, lb, cp, params, kw, variant, device, R):
    """R steps over R independent layer copies."""
    steps = [step_cls(lb, cp, params, kw, variant, device)]
    for _ in range(R - 1):
        nb, np_ = clone_layer(lb, params)
        steps.append(step_cls(nb, cp, np_, kw, variant, device))
    return steps


def capture(fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def dp_max(value, world, device):
    """Max over the ranks of a per-rank time (ms): the step time of the
    data-parallel job is its slowest rank.  world == 1 returns value."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_steps(steps, inputs, W, K, e2e=False, profile=False):
    """W warm-up steps (direct calls), then K timed steps back to back.
    Step i runs on layer copy i % R with inputs[i]: the R copies together
    touch more than twice the L2 per rotation, so every step starts with its
    caches out of L2 (no flush writes needed).  Each timed step is one CUDA
    graph holding all of the step's library calls, captured beforehand; the
    K replays are bracketed by one pair of events after a synchronize.
    e2e: every step also copies its inputs from pinned host memory into the
    device buffers its calls read and copies its output back to pinned host
    memory, all inside the timed region, as a serving loop would: step j's
    graph holds, beside its library calls, a branch on a second stream that
    copies step j+1's inputs in and step j-1's output out (each step has its
    own input buffers, and an output buffer is reused only R steps later), so
    the copies overlap the compute and one graph launch drives a whole step.
    The first step's inputs are copied before the first replay and the last
    output after the last, both inside the timed region.  Returns ms per
    step."""
    import torch
    R = len(steps)
    for i in range(W):
        st = steps[i % R]
        for c in st.calls:
            c(inputs[i])
    torch.cuda.synchronize()
    graphs = []
    outs = None
    if e2e:
        # step j-1's output is copied out while step j computes into another
        # copy's output buffer: at least two output buffers
        assert R >= 2, "the overlapped e2e copies need at least two output buffers"
        outs = [torch.empty_like(steps[i % R].out, device="cpu").pin_memory() for i in range(W, W + K)]
        cs = torch.cuda.Stream()
        for j in range(K):
            i = W + j
            st, x = steps[i % R], inputs[i]
            nxt = inputs[i + 1] if j + 1 < K else None
            prev = (outs[j - 1], steps[(i - 1) % R].out) if j >= 1 else None

            def body(st=st, x=x, nxt=nxt, prev=prev):
                cur = torch.cuda.current_stream()
                fork = torch.cuda.Event()
                fork.record(cur)
                cs.wait_event(fork)
                with torch.cuda.stream(cs):
                    if nxt is not None:
                        for k, v in nxt["host"].items():
                            nxt[k].copy_(v, non_blocking=True)
                    if prev is not None:
                        prev[0].copy_(prev[1], non_blocking=True)
                for c in st.calls:
                    c(x)
                join = torch.cuda.Event()
                join.record(cs)
                cur.wait_event(join)
            graphs.append(capture(body))
    else:
        for i in range(W, W + K):
            st, x = steps[i % R], inputs[i]
            graphs.append(capture(lambda: [c(x) for c in st.calls]))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if profile:
        torch.cuda.profiler.start()
    main = torch.cuda.current_stream()
    e0.record(main)
    if e2e:
        x0 = inputs[W]
        for k, v in x0["host"].items():
            x0[k].copy_(v, non_blocking=True)
        for j in range(K):
            graphs[j].replay()
        outs[K - 1].copy_(steps[(W + K - 1) % R].out, non_blocking=True)
    else:
        for j in range(K):
            graphs[j].replay()
    e1.record(main)
    torch.cuda.synchronize()
    if profile:
        torch.cuda.profiler.stop()
    del graphs
    return e0.elapsed_time(e1) / K


def breakdown(steps, inputs, W, K):
    """Per-call times (ms): each call of each copy captured as its own graph,
    one event pair around each replay (includes one graph launch each, so
    the parts add up to more than the pipelined step)."""
    import torch
    R = len(steps)
    n = len(steps[0].sep_calls)
    graphs = [[capture(lambda c=c, x=inputs[W + r]: c(x)) for c in steps[r].sep_calls] for r in range(R)]
    torch.cuda.synchronize()
    segs = []
    for i in range(K):
        gl = graphs[i % R]
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        ev[0].record()
        for j, g in enumerate(gl):
            g.replay()
            ev[j + 1].record()
        torch.cuda.synchronize()
        segs.append([ev[j].elapsed_time(ev[j + 1]) for j in range(n)])
    del graphs
    return [sum(x[j] for x in segs) / len(segs) for j in range(n)]


def call_time(steps, inputs, W, K, j):
    """Average duration (ms) of call j alone: K calls on the R copies in turn
    (so each call's inputs start out of L2), captured as one CUDA graph so
    the calls follow each other like kernels in a step (launch overlap as in
    the step), one event pair around the replay.  Call j must only read the
    caches."""
    import torch
    R = len(steps)
    g = capture(lambda: [steps[i % R].sep_calls[j](inputs[W + i % R]) for i in range(K)])
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / K


def indexer_traffic(key="csla_indexer_scores"):
    """DRAM bytes per indexer call from the committed ncu summary, if it was
    taken on the current kernel source (else None)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[key]
        h = hashlib.sha256()
        for name in t["sources"]:
            with open(os.path.join(ROOT, name), "rb") as f:
                h.update(f.read())
        return float(t["bytes_per_call"]) if h.hexdigest() == t["sha256"] else None
    except Exception:
        return None


# ------------------------------------------------------------------ CPU oracle baseline
def cpu_baseline(n_steps=3):
    """fp64 oracle on the CSA workload (bounded sample): the oracle builds
    one request's cache from the seeded raw stream, then runs whole decode
    steps (indexer -> top-k -> attention) for as many requests as the host
    has oracle threads (every request reads that one cache, each with its
    own query inputs; the oracle runs requests in parallel).  Returns
    (seconds per step, requests per step)."""
    import numpy as np
    import oracle
    import torch
    from csla_synth import normal, permutation
    from csla_synth import torch_gen
    kw = CSA
    L, D, dI, m = kw["L"], kw["D"], kw["dI"], kw["m"]
    seed = 1
    gamma_kv = (1.0 + 0.1 * normal(seed, "gamma_kv", (D,))).astype(np.float32).astype(np.float64)
    wg = normal(seed, "wg", (D,), std=1.0 / D ** 0.5).astype(np.float32).astype(np.float64)
    gb = normal(seed, "gb", (m,)).astype(np.float32).astype(np.float64)
    wgi = normal(seed, "wgi", (dI,), std=1.0 / dI ** 0.5).astype(np.float32).astype(np.float64)
    gbi = normal(seed, "gbi", (m,)).astype(np.float32).astype(np.float64)
    # raw stream of request 0, rank 0 (same generator as the GPU run), on the host
    kv = torch_gen.normal(seed, "kv/0/0", (L, D), device="cpu").to(torch.bfloat16).double().numpy()
    ki = torch_gen.normal(seed, "idx/0/0", (L, dI), device="cpu").to(torch.bfloat16).double().numpy()
    epp = 128 // m
    pages = L // 128
    bt = permutation(seed, "cpu/pages", pages).astype(np.int32).reshape(1, pages)
    rows = np.zeros((pages, epp, D + 64), np.uint8)
    scales = np.zeros((pages, epp), np.float32)
    kidx = np.zeros((pages, epp, dI), np.uint16)
    for b in range(L // m):
        r, s = oracle.compressed_row(kv[b * m:(b + 1) * m], wg, gb, gamma_kv, b)
        pg = bt[0, b // epp]
        rows[pg, b % epp], scales[pg, b % epp] = r, s
        kidx[pg, b % epp] = oracle.index_key(ki[b * m:(b + 1) * m], wgi, gbi)
    win = np.zeros((1, 128, D + 64), np.uint8)
    wsc = np.zeros((1, 128), np.float32)
    for p in range(L - 128, L):
        win[0, p % 128], wsc[0, p % 128] = oracle.window_row(kv[p], gamma_kv, p)
    nreq = max(1, oracle.num_threads())
    cv = oracle.CacheView(m, D, rows, scales, np.repeat(bt, nreq, axis=0), np.repeat(win, nreq, axis=0),
                          np.repeat(wsc, nreq, axis=0), kidx, dI)
    W = normal(seed, "W_iq_cpu", (kw["HI"] * dI, kw["dc"]), std=1.0 / kw["dc"] ** 0.5)
    sink = normal(seed, "sink", (kw["H"],))
    gq = 1.0 + 0.1 * normal(seed, "gamma_q", (D,))
    times = []
    for s in range(n_steps):
        q = normal(seed, "cpu/q/%d" % s, (nreq, kw["H"], D))
        cq = normal(seed, "cpu/cq/%d" % s, (nreq, kw["dc"]))
        hw = normal(seed, "cpu/hw/%d" % s, (nreq, kw["HI"]))
        t0 = time.perf_counter()
        oracle.csa_decode(cv, list(range(nreq)), [L] * nreq, q, gq, cq, W, hw, sink, kw["HI"], kw["k"])
        times.append(time.perf_counter() - t0)
    return times, nreq


def _filled_cache(m, D, n_entries, L, seed, dI=0):
    """Oracle cache view of one request whose entries (and window rows) are
    quantised rows of N(0,1) content through RMSNorm and RoPE at their
    positions, the distribution the compressor produces; index keys bf16
    N(0,1).  What a step costs does not depend on how the rows were made."""
    import numpy as np
    import oracle
    from csla_synth import normal, to_bf16_bits
    epp = 128 // m
    pages = -(-n_entries // epp)
    gamma = (1.0 + 0.1 * normal(seed, "cpu/gamma", (D,))).astype(np.float32).astype(np.float64)
    rb = oracle.row_bytes(D)
    rows = np.zeros((pages, epp, rb), np.uint8)
    scales = np.zeros((pages, epp), np.float32)
    x = normal(seed, "cpu/rows", (n_entries, D))
    for e in range(n_entries):
        rows[e // epp, e % epp], scales[e // epp, e % epp] = oracle.window_row(x[e], gamma, e * m)
    win = np.zeros((1, 128, rb), np.uint8)
    wsc = np.zeros((1, 128), np.float32)
    xw = normal(seed, "cpu/win", (128, D))
    for i, p in enumerate(range(L - 128, L)):
        win[0, p % 128], wsc[0, p % 128] = oracle.window_row(xw[i], gamma, p)
    kidx = to_bf16_bits(normal(seed, "cpu/kidx", (pages, epp, dI))) if dI else None
    bt = np.arange(pages, dtype=np.int32).reshape(1, pages)
    return oracle.CacheView(m, D, rows, scales, bt, win, wsc, kidx, dI)


def cpu_baseline_hca(n_steps=3):
    """fp64 oracle decode steps of the HCA workload (context 2^20 - 64: 8191
    entries + 128 window rows per request and step), one request per oracle
    thread, all reading one cache; (seconds per step, requests per step)."""
    import oracle
    from csla_synth import normal
    kw, seed = HCA, 2
    L = kw["L"] - 64
    import numpy as np
    cv = _filled_cache(kw["m"], kw["D"], L // kw["m"], L, seed)
    nreq = max(1, oracle.num_threads())
    cv = oracle.CacheView(cv.m, cv.D, cv.rows, cv.scales, np.repeat(cv.block_table, nreq, axis=0),
                          np.repeat(cv.win_rows, nreq, axis=0), np.repeat(cv.win_scales, nreq, axis=0), None, 0)
    sink = normal(seed, "sink", (kw["H"],))
    gq = 1.0 + 0.1 * normal(seed, "gamma_q", (kw["D"],))
    times = []
    for s_ in range(n_steps):
        q = normal(seed, "cpu/q/%d" % s_, (nreq, kw["H"], kw["D"]))
        t0 = time.perf_counter()
        oracle.hca_decode(cv, list(range(nreq)), [L] * nreq, q, gq, sink)
        times.append(time.perf_counter() - t0)
    return times, nreq


def cpu_baseline_prefill(n_q=16):
    """fp64 oracle on a sample of the prefill chunk's queries (n_q of the
    4096, spread over the chunk; each query = indexer over its ~66K visible
    entries, top-k 1024, attention over 1152 rows), the oracle's threads
    across queries.  Returns (seconds for the sample, threads)."""
    import numpy as np
    import oracle
    from csla_synth import normal
    kw, seed = PREFILL, 4
    L1 = kw["L0"] + kw["T"]
    cv = _filled_cache(kw["m"], kw["D"], L1 // kw["m"], L1, seed, dI=kw["dI"])
    W = normal(seed, "W_iq_cpu", (kw["HI"] * kw["dI"], kw["dc"]), std=1.0 / kw["dc"] ** 0.5)
    sink = normal(seed, "sink", (kw["H"],))
    gq = 1.0 + 0.1 * normal(seed, "gamma_q", (kw["D"],))
    lens = [kw["L0"] + 1 + (i * kw["T"]) // n_q for i in range(n_q)]
    q = normal(seed, "cpu/pq", (n_q, kw["H"], kw["D"]))
    cq = normal(seed, "cpu/pcq", (n_q, kw["dc"]))
    hw = normal(seed, "cpu/phw", (n_q, kw["HI"]))
    t0 = time.perf_counter()
    oracle.csa_decode(cv, np.zeros(n_q, np.int32), lens, q, gq, cq, W, hw, sink, kw["HI"], kw["k"])
    return time.perf_counter() - t0, min(n_q, oracle.num_threads())


def run_reference(args):
    t_setup = time.perf_counter()
    times, nreq = cpu_baseline(n_steps=args.warmup + args.steps)
    timed = times[args.warmup:]
    per_step = sum(timed) / len(timed)
    value = nreq / per_step
    sample = ("%d requests of the CSA workload per step (context 131072, 32768 entries, k=512; one oracle-built "
              "cache read by all), fp64 oracle, one host thread per request" % nreq)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded splitmix64 / Box-Muller)",
            "config": {"workload": "csa_decode_B8_L131072", "sample": "%d requests per step" % nreq},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nreq, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "setup_s": time.perf_counter() - t_setup}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main
def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return

    import torch
    import torch.distributed as dist
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "csla_build", os.path.join(ROOT, "compressed_sparse_long_append_b200", "build.py"))
    cbuild = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(cbuild)
    cbuild.build()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    W, K = max(3, args.warmup), args.steps
    seed = 1
    if args.prefill_only or args.hca_only or args.e4m3_only:
        if args.prefill_only:
            key, res = "csa_prefill", prefill_leg(W, K, seed + 2, rank, world, device, args.variant,
                                                  profile=args.profile)
        elif args.hca_only:
            key, res = "hca_decode", hca_leg(W, K, seed + 1, rank, world, device, args.variant, peaks()[0],
                                             profile=args.profile)
        else:
            key, res = "csa_decode_e4m3_keys", e4m3_leg(W, K, seed, rank, world, device, args.variant,
                                                        profile=args.profile)
        if rank == 0:
            print(json.dumps({key: res}), flush=True)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    # ---------------- CSA layer (the headline workload)
    kw = dict(CSA)
    R, m, B = CSA_COPIES, kw["m"], kw["B"]
    # request b starts b % m tokens short, so B/m requests close a block every step
    before = -(-(W + K) // R)
    L0s = [kw["L"] - before - (b % m) for b in range(B)]
    lb, cp, params = build_layer(kw, B, L0s, seed, rank, device)
    inputs = step_inputs(kw, B, W + K, seed, rank, device)
    CsaStep.fused = args.fused_step
    steps = make_copies(CsaStep, lb, cp, params, kw, args.variant, device, R)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(local)
    clk.start()
    ms_step = run_steps(steps, inputs, W, K, profile=args.profile)
    clocks = clk.stop()
    if world > 1:
        dist.barrier()
    ms_step = dp_max(ms_step, world, device)

    if args.profile:
        args.no_hca = args.no_cpu_baseline = True
        ms_e2e, h2d, d2h, seg, ms_idx = float("nan"), 0, 0, [float("nan")] * 4, float("nan")
    else:
        # e2e: the same steps again (contexts grow by another K/R tokens), host buffers
        ms_e2e = run_steps(steps, inputs, W, K, e2e=True)
        h2d = sum(v.numel() * v.element_size() for k, v in inputs[0]["host"].items())
        d2h = steps[0].out.numel() * steps[0].out.element_size()
        seg = breakdown(steps, inputs, W, K)
        ms_idx = call_time(steps, inputs, W, K, 1)
    ms_e2e = dp_max(ms_e2e, world, device)

    # algorithmic bytes of one indexer call: every visible key (dI bf16) read
    # once, one f32 score written per key, W_iq read once
    nv = sum(int(x) // m for st in steps for x in st.lb.len.tolist()) / R
    idx_bytes = nv * (kw["dI"] * 2 + 4) + kw["HI"] * kw["dI"] * kw["dc"] * 2
    peak, peak_kind = peaks()
    achieved = idx_bytes / (ms_idx * 1e-3) / 1e9

    hca = None
    if not args.no_hca:
        del steps, lb
        torch.cuda.empty_cache()
        hca = hca_leg(W, K, seed + 1, rank, world, device, args.variant, peak)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            try:
                ht, nreq = cpu_baseline_hca(3)
                hca["cpu_baseline"] = {"value": nreq / (sum(ht) / len(ht)), "unit": UNIT, "cores": nreq,
                                       "kind": "oracle",
                                       "sample": "%d requests of this workload (context 2^20 - 64, 8191 entries + "
                                                 "128 window rows; one cache read by all), 3 decode steps, fp64 "
                                                 "oracle, one thread per request" % nreq}
            except Exception as e:  # the baseline never blocks the GPU line
                hca["cpu_baseline"] = {"value": None, "unit": UNIT, "cores": 0, "kind": "oracle",
                                       "sample": "failed: %s" % e}

    pre = None
    if not args.no_prefill and not args.profile:
        if args.no_hca:
            del steps, lb
            torch.cuda.empty_cache()
        pre = prefill_leg(W, K, seed + 2, rank, world, device, args.variant)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            try:
                pt, thr = cpu_baseline_prefill(16)
                pre["cpu_baseline"] = {"value": 16 / pt, "unit": "tokens/s", "cores": thr, "kind": "oracle",
                                       "sample": "16 of the chunk's 4096 queries (spread over it) against a "
                                                 "cache of the same size, fp64 oracle, threads across queries"}
            except Exception as e:  # the baseline never blocks the GPU line
                pre["cpu_baseline"] = {"value": None, "unit": "tokens/s", "cores": 0, "kind": "oracle",
                                       "sample": "failed: %s" % e}
    if args.no_hca and args.no_prefill and not args.profile:
        del steps, lb
        torch.cuda.empty_cache()
    e4 = None
    if not args.no_e4m3 and not args.profile:
        e4 = e4m3_leg(W, K, seed, rank, world, device, args.variant)
    inv = None
    if not args.no_invariance and not args.profile:
        inv = invariance_leg(W, K, seed + 4, rank, world, device, args.variant)
    stk = None
    if not args.no_stack and not args.profile:
        stk = stack_leg(W, K, seed + 6, rank, world, device, args.variant, args.stack_layers)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            ct, nreq = cpu_baseline(n_steps=3)
            v = nreq / (sum(ct) / len(ct))
            cpu = {"value": v, "unit": UNIT, "cores": nreq, "kind": "oracle",
                   "sample": "%d requests of this workload (context 131072, k=512; one oracle-built cache read "
                             "by all), 3 decode steps, fp64 oracle, one thread per request" % nreq}
        except Exception as e:  # the baseline never blocks the GPU line
            cpu = {"value": None, "unit": UNIT, "cores": 0, "kind": "oracle", "sample": "failed: %s" % e}

    if rank == 0:
        launches_per_step = csa_launches(kw, args.variant, CsaStep.fused)
        line = {
            "metric": METRIC, "value": B * world / (ms_step * 1e-3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded splitmix64 / Box-Muller token streams, caches built by csla_compress_append)",
            "config": {"workload": "csa_decode_B8_L131072", "requests_per_gpu": B, "context": kw["L"],
                       "context_stagger": "request b is b %% %d tokens shorter: %d of %d requests close a "
                                          "block every step" % (m, B // m, B),
                       "m": 4, "compressed_entries": kw["L"] // 4, "heads": 64, "head_dim": 512,
                       "index_heads": 16, "index_dim": 128, "dc": 1024, "topk": 512, "window": 128,
                       "l2": "inputs larger than L2: %d rotating copies of the layer (caches + W_iq), "
                             "~%d MB touched per rotation vs 126 MB L2" % (R, R * 75),
                       "launch": ("one CUDA graph per step (csla_csa_decode_step: the append on a side stream "
                                  "beside the indexer's scoring of the entries already complete)" if CsaStep.fused else
                                  "one CUDA graph per step (the four library calls)") +
                                 ", K graphs replayed back to back between one event pair",
                       "parallelism": "dp%d over requests" % world, "variant": args.variant},
            "segments_ms": {"compress_append": seg[0], "indexer_scores": seg[1], "topk_select": seg[2],
                            "csa_attend": seg[3], "note": "one graph launch per call, serialised"},
            "roofline": {"bound": "hbm", "kernel": "csla_indexer_scores (iq_project + indexer)",
                         "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_kind": peak_kind, "traffic": indexer_traffic(),
                         "algorithmic_bytes": idx_bytes, "call_ms": ms_idx},
            "cpu_baseline": cpu,
            "e2e": {"value": B * world / (ms_e2e * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * K,
            "clocks": clocks,
            "hca_decode": hca,
            "csa_prefill": pre,
            "csa_decode_e4m3_keys": e4,
            "invariance_decode": inv,
            "stack_decode": stk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
