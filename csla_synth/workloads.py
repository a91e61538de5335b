"""Workload shapes and seeded input recipes (no method arithmetic).

Each configuration below is one of the benchmark / parity workloads of the
CSA/HCA decode path; the recipe states which seeded stream feeds each tensor.
"""
from dataclasses import dataclass, field

import numpy as np

from . import normal, to_bf16_bits


@dataclass(frozen=True)
class Workload:
    name: str
    B: int            # requests in the batch
    L: int            # context length (tokens so far, current one included)
    m: int            # compression ratio (4 = CSA, 128 = HCA)
    H: int            # query heads
    D: int            # head dim (last d_rope dims carry RoPE)
    HI: int = 0       # index heads (CSA only)
    dI: int = 0       # index head dim
    dc: int = 0       # query latent dim
    k: int = 0        # top-k (CSA only)
    n_win: int = 128
    d_rope: int = 64
    theta: float = 10000.0
    eps: float = 1e-6
    act_bf16: bool = True   # activations are exact bf16 values
    seed: int = 0
    key_fmt: int = 0        # CSA index keys: 0 bf16, 1 E4M3 codes + per-entry power-of-two scale
    gate: int = 0           # compressor gate: 0 one per token, 1 one per token and channel

    @property
    def is_csa(self):
        return self.k > 0


# configs of the contract
CSA_TINY = Workload("csa_decode_tiny_L2048", B=1, L=2048, m=4, H=8, D=128, HI=4, dI=64, dc=128,
                    k=64, act_bf16=False, seed=0)
CSA_DECODE = Workload("csa_decode_B8_L131072", B=8, L=131072, m=4, H=64, D=512, HI=16, dI=128,
                      dc=1024, k=512, seed=1)
HCA_DECODE = Workload("hca_decode_B4_L1048576", B=4, L=1048576, m=128, H=64, D=512, seed=2)
# prefill chunk: T = 4096 new tokens (and queries) after a 262144-token prefix,
# so the last query sees 66560 compressed entries; B counts queries here
CSA_PREFILL = Workload("csa_prefill_T4096_L262144", B=4096, L=262144 + 4096, m=4, H=64, D=512, HI=16,
                       dI=128, dc=1024, k=1024, seed=4)


def _act(w: Workload, name, shape, std=1.0, start=0):
    x = normal(w.seed, name, shape, std=std, start=start)
    if w.act_bf16:
        from . import bf16_bits_to_f64
        x = bf16_bits_to_f64(to_bf16_bits(x))
    return x


def layer_params(w: Workload):
    """Per-layer parameters (float64 arrays; exact bf16 values for bf16 runs
    are not needed: parameters are fp32 inputs of the kernels)."""
    p = {
        "gamma_kv": 1.0 + 0.1 * normal(w.seed, "gamma_kv", (w.D,)),
        "gamma_q": 1.0 + 0.1 * normal(w.seed, "gamma_q", (w.D,)),
        "wg": normal(w.seed, "wg", (w.D,), std=1.0 / np.sqrt(w.D)),
        "gb": normal(w.seed, "gb", (w.m,)),
        "sink": normal(w.seed, "sink", (w.H,)),
    }
    if w.is_csa:
        p["wgi"] = normal(w.seed, "wgi", (w.dI,), std=1.0 / np.sqrt(w.dI))
        p["gbi"] = normal(w.seed, "gbi", (w.m,))
    if w.gate == 1:
        # per-channel gate x_id * w_d + b_id: an O(1) weight per channel and
        # a bias per position and channel
        p["wg"] = normal(w.seed, "wg_ch", (w.D,))
        p["gb"] = normal(w.seed, "gb_ch", (w.m, w.D))
        if w.is_csa:
            p["wgi"] = normal(w.seed, "wgi_ch", (w.dI,))
            p["gbi"] = normal(w.seed, "gbi_ch", (w.m, w.dI))
    if w.is_csa:
        p["W_iq"] = _act(w, "W_iq", (w.HI * w.dI, w.dc), std=1.0 / np.sqrt(w.dc))
    # fp32 parameters: round once so both sides see the same fp32 values
    return {k: v.astype(np.float32).astype(np.float64) for k, v in p.items()}


def token_stream(w: Workload, req, start, stop):
    """Raw per-token KV (and index-key) hidden states of request `req` at
    positions start..stop-1: rows start..stop-1 of the streams "kv/<req>" and
    "idx/<req>" (element p*width + d of the stream is dim d of position p)."""
    n = stop - start
    out = {"kv": _act(w, "kv/%d" % req, (n, w.D), start=start * w.D)}
    if w.is_csa:
        out["idx"] = _act(w, "idx/%d" % req, (n, w.dI), start=start * w.dI)
    return out


def step_inputs(w: Workload, step):
    """Per-step query-side inputs of a decode step."""
    out = {
        "q": _act(w, "q/%d" % step, (w.B, w.H, w.D)),
    }
    if w.is_csa:
        out["cq"] = _act(w, "cq/%d" % step, (w.B, w.dc))
        out["head_w"] = normal(w.seed, "head_w/%d" % step, (w.B, w.HI)).astype(np.float32) \
            .astype(np.float64)
    return out


def prefill_inputs(w: Workload, T, tag=0):
    """Query-side inputs of T prefill queries (one per new token)."""
    out = {"q": _act(w, "pq/%d" % tag, (T, w.H, w.D))}
    if w.is_csa:
        out["cq"] = _act(w, "pcq/%d" % tag, (T, w.dc))
        out["head_w"] = normal(w.seed, "phw/%d" % tag, (T, w.HI)).astype(np.float32).astype(np.float64)
    return out
