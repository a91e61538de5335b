"""Context-parallel prefill of one long request over R ranks (haiqwa
"DeepSeek-V4" blog, §百万 token 怎么切分到多张卡).

The request's tokens 0..N-1 are split into contiguous ranges [p_r, p_r+1),
one per rank.  Two communication stages:

1. Boundary exchange.  Rank r sends rank r+1 the raw input rows that rank
   r+1 needs but does not hold: the open compression block at p_r+1 (so that
   no block is cut at the rank boundary) and the n_win-1 positions before
   p_r+1 (the sliding window of the first queries of rank r+1).  These are
   positions [a_r+1, p_r+1) with a_r+1 block-aligned.  Rank r+1 appends them
   to a state whose length is set to a_r+1 (an empty tail), then appends its
   own tokens: it now holds the compressed entries of every block that
   closes in its range, and the window rows of its queries.  The pages send
   the last m raw entries; the window rows are this library's addition (the
   pages do not discuss the sliding-window branch under CP).  The exchange
   moves inputs only, so no rank waits for another's compute.
2. All-gather and reassembly.  Every rank packs the entries of the blocks
   that close in its range into a fixed-length run of records padded with
   zero records (csla_cp_select), one all-gather of the equal-sized runs
   gives every rank all runs, and csla_cp_place writes each rank's valid
   records into the paged cache at their global block index (the
   select-and-pad step: padding dropped, entries in block order).

Then each rank answers its own queries (positions p_r .. p_r+1 - 1) with
per-row visible lengths (a query sees what a decode step at its position
sees), in chunks of at most q_chunk rows.  After the call every rank holds
the request's full compressed cache; the window ring, tail and length of the
request are those of the last rank.

This module holds the plan (pure integer bookkeeping), the rank-local steps
on the library (LibRank), the distributed driver (run_cp_prefill, over any
torch.distributed backend) and a single-process driver that runs the ranks
one after another with the collectives replaced by tensor copies
(run_cp_prefill_local).
"""
from dataclasses import dataclass


@dataclass(frozen=True)
class CpPlan:
    """Token ranges and block bookkeeping of a CP prefill of N tokens."""
    N: int
    m: int
    n_win: int
    starts: tuple   # p_0 = 0 < p_1 < ... < p_R = N

    @property
    def R(self):
        return len(self.starts) - 1

    def rng(self, r):
        return self.starts[r], self.starts[r + 1]

    def bnd_start(self, r):
        """First boundary position a_r received by rank r (a_0 = 0: none)."""
        p = self.starts[r]
        if r == 0:
            return p
        return max(0, (p - (self.n_win - 1)) // self.m * self.m)

    def n_bnd(self, r):
        return self.starts[r] - self.bnd_start(r)

    def bnd_offset(self, r):
        """Offset, within rank r's own rows, of the rows rank r+1 receives."""
        return self.bnd_start(r + 1) - self.starts[r]

    def blocks(self, r):
        """(first block, count) of the blocks that close in rank r's range."""
        p0, p1 = self.rng(r)
        return p0 // self.m, p1 // self.m - p0 // self.m

    @property
    def E_max(self):
        return max(max(self.blocks(r)[1] for r in range(self.R)), 1)

    @property
    def head_rows(self):
        """Token-row buffer rows ahead of a rank's own tokens (boundary rows)."""
        return self.n_win + self.m - 2


def cp_plan(N, R, m, n_win=128, starts=None):
    """Even split of N tokens over R ranks (or the given starts).  Every
    rank's boundary rows must lie inside the previous rank's range."""
    if starts is None:
        starts = [N * r // R for r in range(R + 1)]
    starts = tuple(int(x) for x in starts)
    if len(starts) != R + 1 or starts[0] != 0 or starts[-1] != N:
        raise ValueError("starts must run from 0 to N in R steps")
    if any(b <= a for a, b in zip(starts, starts[1:])):
        raise ValueError("every rank needs at least one token")
    plan = CpPlan(N, m, n_win, starts)
    for r in range(1, R):
        if plan.bnd_start(r) < starts[r - 1]:
            raise ValueError("rank %d's range is shorter than the boundary it sends (%d rows)"
                             % (r - 1, plan.n_bnd(r)))
    return plan


class LibRank:
    """Rank r's steps on the library, for one request in slot `slot` of the
    layer buffers `lb` (a full-size paged cache; the block table must map
    every page of the request)."""

    def __init__(self, plan: CpPlan, r, lb, cp, slot=0, device="cuda"):
        import torch
        from . import csla as C
        self.C, self.plan, self.r, self.lb, self.cp = C, plan, r, lb, cp
        self.slot = slot
        self.cfg = lb.cfg()
        p0, p1 = plan.rng(r)
        self.T = p1 - p0
        rb = lb.shape.row_bytes
        H0 = plan.head_rows
        self.buf = torch.zeros((H0 + self.T, rb), dtype=torch.uint8, device=device)
        self.bufsc = torch.zeros(H0 + self.T, dtype=torch.float32, device=device)
        self.rec = C.csla_cp_record_bytes(self.cfg)
        self.send = torch.zeros((plan.E_max, self.rec), dtype=torch.uint8, device=device)
        self.slots1 = torch.tensor([slot], dtype=torch.int32, device=device)
        self.device = device

    # -- stage 1
    def boundary_out(self, kv, kidx=None):
        """Rows of this rank's input that rank r+1 needs (views of kv/kidx)."""
        a = self.plan.bnd_offset(self.r)
        return kv[a:], (kidx[a:] if kidx is not None else None)

    def compress(self, bkv, bkidx, kv, kidx):
        """Append the received boundary rows (positions a_r..p_r-1) to an
        empty-tailed state at a_r, then this rank's own tokens."""
        C, plan, r = self.C, self.plan, self.r
        dt = C.CSLA_BF16 if kv.element_size() == 2 else C.CSLA_F32   # bf16 or f32 rows
        H0 = plan.head_rows
        self.lb.len[self.slot] = plan.bnd_start(r)
        nb = plan.n_bnd(r)
        st, cache, cps = self.lb.state(), self.lb.cache(), self.cp.struct()
        stride = H0 + self.T
        if nb > 0:
            tok = C.token_rows(self.buf, self.bufsc, stride, H0 - nb)
            C.csla_compress_append(self.cfg, st, cache, self.slots1, 1, nb, bkv, bkidx, dt, cps, tok=tok)
        tok = C.token_rows(self.buf, self.bufsc, stride, H0)
        C.csla_compress_append(self.cfg, st, cache, self.slots1, 1, self.T, kv, kidx, dt, cps, tok=tok)

    # -- stage 2
    def select(self):
        b_lo, n = self.plan.blocks(self.r)
        self.C.csla_cp_select(self.cfg, self.lb.state(), self.lb.cache(), self.slot, b_lo, n, self.plan.E_max,
                              self.send)
        return self.send

    def place(self, recv):
        """recv: [R][E_max][record] uint8, every rank's run."""
        R = self.plan.R
        b = [self.plan.blocks(q) for q in range(R)]
        self.C.csla_cp_place(self.cfg, self.lb.state(), self.lb.cache(), self.slot, recv, self.plan.E_max,
                             [x[0] for x in b], [x[1] for x in b])

    # -- queries
    def queries(self, q, sink, gamma_q, out, cq=None, W_iq=None, head_w=None, k=0, q_chunk=1024,
                variant=0, idx_out=None):
        """This rank's T queries (positions p_r ..), q [T][H][D] and, for
        CSA, cq [T][dc], head_w [T][HI] f32; out [T][H][D].  idx_out: an
        optional [T][k] int32 tensor that receives the CSA top-k lists."""
        import torch
        C, plan = self.C, self.plan
        p0, p1 = plan.rng(self.r)
        H0 = plan.head_rows
        dt = C.CSLA_BF16 if q.element_size() == 2 else C.CSLA_F32
        odt = C.CSLA_BF16 if out.element_size() == 2 else C.CSLA_F32
        st, cache = self.lb.state(), self.lb.cache()
        csa = self.lb.shape.is_csa
        m = plan.m
        for c0 in range(0, self.T, q_chunk):
            c1 = min(self.T, c0 + q_chunk)
            n = c1 - c0
            q_len = torch.arange(p0 + c0 + 1, p0 + c1 + 1, dtype=torch.int32, device=self.device)
            base = torch.full((n,), H0 - p0, dtype=torch.int32, device=self.device)
            rows_slots = torch.full((n,), self.slot, dtype=torch.int32, device=self.device)
            qs_att = C.queries(q_len, self.buf, self.bufsc, base, H0 + self.T)
            max_len = p0 + c1
            if csa:
                qs_rows = C.queries(q_len, one_request=True)
                stride = max_len // m
                scores = torch.empty((n, max(stride, 1)), dtype=torch.float32, device=self.device)
                idx = idx_out[c0:c1] if idx_out is not None else \
                    torch.empty((n, k), dtype=torch.int32, device=self.device)
                wsi = C.csla_workspace_size(self.cfg, C.CSLA_OP_INDEXER, n, max_len)
                wsa = C.csla_workspace_size(self.cfg, C.CSLA_OP_CSA_ATTEND, n, k)
                ws_i = torch.empty(max(wsi, 16), dtype=torch.uint8, device=self.device)
                ws_a = torch.empty(max(wsa, 16), dtype=torch.uint8, device=self.device)
                cdt = C.CSLA_BF16 if cq.element_size() == 2 else C.CSLA_F32
                wdt = C.CSLA_BF16 if W_iq.element_size() == 2 else C.CSLA_F32
                C.csla_indexer_scores(self.cfg, st, cache, rows_slots, n, max_len, cq[c0:c1], cdt, W_iq, wdt,
                                      head_w[c0:c1], scores, max(stride, 1), ws_i, wsi, qs=qs_rows)
                C.csla_topk_select(self.cfg, st, rows_slots, n, max_len, scores, max(stride, 1), k, idx,
                                   qs=qs_rows)
                C.csla_csa_attend(self.cfg, st, cache, rows_slots, n, q[c0:c1], dt, idx, k, sink, gamma_q,
                                  out[c0:c1], odt, variant, ws_a, wsa, qs=qs_att)
            else:
                wsa = C.csla_workspace_size(self.cfg, C.CSLA_OP_HCA_ATTEND, n, max_len)
                ws_a = torch.empty(max(wsa, 16), dtype=torch.uint8, device=self.device)
                C.csla_hca_attend(self.cfg, st, cache, rows_slots, n, max_len, q[c0:c1], dt, sink, gamma_q,
                                  out[c0:c1], odt, variant, ws_a, wsa, qs=qs_att)
        return out


def _bnd_shapes(plan, r, kv_like, kidx_like):
    """Empty tensors for the boundary rows rank r receives."""
    import torch
    nb = plan.n_bnd(r)
    bkv = torch.empty((nb,) + tuple(kv_like.shape[1:]), dtype=kv_like.dtype, device=kv_like.device)
    bki = None if kidx_like is None else torch.empty((nb,) + tuple(kidx_like.shape[1:]), dtype=kidx_like.dtype,
                                                     device=kidx_like.device)
    return bkv, bki


def run_cp_prefill(rank_obj, kv, kidx=None, group=None):
    """Stages 1 and 2 on this process's rank (torch.distributed, any backend
    whose tensors rank_obj uses).  Every rank calls it; afterwards
    rank_obj.queries answers the rank's queries."""
    import torch
    import torch.distributed as dist
    plan, r = rank_obj.plan, rank_obj.r
    R = plan.R
    assert dist.get_world_size(group) == R and dist.get_rank(group) == r
    reqs = []
    if r + 1 < R:
        okv, oki = rank_obj.boundary_out(kv, kidx)
        okv = okv.contiguous()
        reqs.append(dist.isend(okv, r + 1, group=group))
        if oki is not None:
            oki = oki.contiguous()
            reqs.append(dist.isend(oki, r + 1, group=group))
    bkv = bki = None
    if r > 0:
        bkv, bki = _bnd_shapes(plan, r, kv, kidx)
        reqs.append(dist.irecv(bkv, r - 1, group=group))
        if bki is not None:
            reqs.append(dist.irecv(bki, r - 1, group=group))
    for q in reqs:
        q.wait()
    rank_obj.compress(bkv, bki, kv, kidx)
    send = rank_obj.select()
    parts = [torch.empty_like(send) for _ in range(R)]
    dist.all_gather(parts, send, group=group)
    rank_obj.place(torch.stack(parts))
    return rank_obj


def run_cp_prefill_local(ranks, kvs, kidxs=None):
    """The same stages for all ranks in one process, one after another; the
    point-to-point sends and the all-gather become tensor copies."""
    import torch
    R = len(ranks)
    kidxs = kidxs if kidxs is not None else [None] * R
    bnd = [(None, None)]
    for r in range(R - 1):
        okv, oki = ranks[r].boundary_out(kvs[r], kidxs[r])
        bnd.append((okv.clone(), None if oki is None else oki.clone()))
    for r in range(R):
        ranks[r].compress(bnd[r][0], bnd[r][1], kvs[r], kidxs[r])
    recv = torch.stack([ranks[r].select().clone() for r in range(R)])
    for r in range(R):
        ranks[r].place(recv)
    return ranks
