"""Device buffers of one CSA or HCA layer, owned by torch, described to the
library through the csla_cache / csla_state structs.

Plumbing only: this module allocates and zero-fills memory and builds the
ctypes structs; all computation happens in libcsla's kernels.
"""
from dataclasses import dataclass

import torch

from . import csla as C


@dataclass(frozen=True)
class LayerShape:
    m: int                 # 4 (CSA) or 128 (HCA)
    D: int = 512
    H: int = 64
    HI: int = 16
    dI: int = 128
    dc: int = 1024
    n_win: int = 128
    d_rope: int = 64
    theta: float = 10000.0
    eps: float = 1e-6
    key_fmt: int = C.CSLA_KEY_BF16   # CSA index keys: bf16, or E4M3 codes + per-entry power-of-two scale
    gate: int = C.CSLA_GATE_TOKEN    # compressor gate: one per token, or one per token and channel

    @property
    def is_csa(self):
        return self.m == 4

    @property
    def row_bytes(self):
        return (self.D - self.d_rope) + 2 * self.d_rope

    @property
    def epp(self):
        return C.CSLA_PAGE_TOKENS // self.m

    def cfg(self):
        return C.csla_cfg(self.m, self.D, self.d_rope, self.H, self.HI if self.is_csa else 0,
                          self.dI if self.is_csa else 0, self.dc if self.is_csa else 0, self.n_win,
                          self.theta, self.eps, self.key_fmt if self.is_csa else C.CSLA_KEY_BF16, self.gate)


class LayerBuffers:
    """Classical cache pages + block table + state cache for `n_slots` requests.
    `block_table` ([n_slots, bt_stride] int32 on the device) is used as given
    instead of a table of the layer's own (layers of one model share one)."""

    def __init__(self, shape: LayerShape, n_slots: int, n_pages: int, bt_stride: int, device="cuda",
                 block_table=None):
        s = shape
        self.shape = s
        self.device = torch.device(device)
        dev = self.device
        self.rows = torch.zeros((n_pages, s.epp, s.row_bytes), dtype=torch.uint8, device=dev)
        self.scales = torch.zeros((n_pages, s.epp), dtype=torch.float32, device=dev)
        fp8_keys = s.is_csa and s.key_fmt == C.CSLA_KEY_E4M3
        kdt = torch.uint8 if fp8_keys else torch.int16
        self.kidx = torch.zeros((n_pages, s.epp, s.dI), dtype=kdt, device=dev) if s.is_csa else None
        self.kscale = torch.zeros((n_pages, s.epp), dtype=torch.float32, device=dev) if fp8_keys else None
        if block_table is None:
            block_table = torch.full((n_slots, bt_stride), -1, dtype=torch.int32, device=dev)
        elif (block_table.dtype != torch.int32 or tuple(block_table.shape) != (n_slots, bt_stride)
              or not block_table.is_contiguous() or block_table.device.type != dev.type):
            raise ValueError("block_table must be a contiguous [n_slots, bt_stride] int32 tensor on %s" % dev)
        self.block_table = block_table
        self.win_rows = torch.zeros((n_slots, s.n_win, s.row_bytes), dtype=torch.uint8, device=dev)
        self.win_scales = torch.zeros((n_slots, s.n_win), dtype=torch.float32, device=dev)
        self.tail_kv = torch.zeros((n_slots, s.m, s.D), dtype=torch.float32, device=dev)
        self.tail_idx = torch.zeros((n_slots, s.m, s.dI), dtype=torch.float32, device=dev) if s.is_csa else None
        self.len = torch.zeros((n_slots,), dtype=torch.int32, device=dev)
        self.n_slots, self.n_pages, self.bt_stride = n_slots, n_pages, bt_stride
        self._cfg = s.cfg()

    def cfg(self):
        return self._cfg

    def cache(self):
        return C.csla_cache(self.rows.data_ptr(), self.scales.data_ptr(),
                            self.kidx.data_ptr() if self.kidx is not None else None,
                            self.block_table.data_ptr(), self.bt_stride, self.n_pages,
                            self.kscale.data_ptr() if self.kscale is not None else None)

    def state(self):
        return C.csla_state(self.win_rows.data_ptr(), self.win_scales.data_ptr(), self.tail_kv.data_ptr(),
                            self.tail_idx.data_ptr() if self.tail_idx is not None else None,
                            self.len.data_ptr(), self.n_slots)

    def host_view(self):
        """Host copies of every buffer (for checks against an independent model)."""
        out = {k: getattr(self, k).cpu().numpy() for k in
               ("rows", "scales", "block_table", "win_rows", "win_scales", "tail_kv", "len")}
        if self.kidx is not None:
            out["kidx"] = self.kidx.cpu().numpy() if self.kscale is not None else self.kidx.cpu().numpy().view("uint16")
            out["tail_idx"] = self.tail_idx.cpu().numpy()
        if self.kscale is not None:
            out["kscale"] = self.kscale.cpu().numpy()
        return out


class LayerStack:
    """The attention layers of one model over one block table.  A page is
    128 raw tokens of a request in every layer (32 CSA entries or 1 HCA
    entry), so page id p of a request names page p of each layer's own
    pool: one allocation covers the whole stack.  Every layer keeps its own
    pools, window ring, tail and length (each layer appends its own
    compressed KV).  `shapes[i]` is layer i's shape, e.g. CSA and HCA
    layers interleaved."""

    def __init__(self, shapes, n_slots: int, n_pages: int, bt_stride: int, device="cuda"):
        self.device = torch.device(device)
        self.block_table = torch.full((n_slots, bt_stride), -1, dtype=torch.int32, device=self.device)
        self.layers = [LayerBuffers(s, n_slots, n_pages, bt_stride, device, block_table=self.block_table)
                       for s in shapes]
        self.n_slots, self.n_pages, self.bt_stride = n_slots, n_pages, bt_stride

    def __len__(self):
        return len(self.layers)

    def __getitem__(self, i):
        return self.layers[i]


class CompressParams:
    """fp32 compressor parameters on the device."""

    def __init__(self, gamma_kv, wg, gb, wgi=None, gbi=None, device="cuda"):
        f = lambda x: None if x is None else torch.as_tensor(x, dtype=torch.float32).to(device).contiguous()
        self.gamma_kv, self.wg, self.gb, self.wgi, self.gbi = f(gamma_kv), f(wg), f(gb), f(wgi), f(gbi)

    def struct(self):
        p = lambda t: None if t is None else t.data_ptr()
        return C.csla_compress_params(p(self.gamma_kv), p(self.wg), p(self.gb), p(self.wgi), p(self.gbi))


def dtype_code(t: torch.Tensor):
    if t.dtype == torch.float32:
        return C.CSLA_F32
    if t.dtype == torch.bfloat16:
        return C.CSLA_BF16
    raise TypeError("unsupported dtype %s" % t.dtype)
