"""The exactness argument of the fused indexer + top-k, checked on the CPU
against the oracle's top-k rule (largest scores, ties to the lower index,
ascending output): when at least k scores reach a threshold t0, the top-k
taken among those candidates alone equals the top-k over the whole row,
whatever t0 is; otherwise the call falls back to the whole row.  t0 here
comes from the same kind of sample the library takes (32 pages of 32
entries, evenly spaced), on rows with heavy ties, signed zeros and a rising
trend."""
import numpy as np
import pytest

import oracle
from csla_synth import integers, normal


def sample_threshold(s, k, pages=32, page=32):
    """r-th largest of an evenly spaced page sample, r scaled to the row."""
    n = len(s)
    Z = max(1, -(-(-(-n // page)) // pages))
    idx = [p * Z * page + i for p in range(pages) for i in range(page) if p * Z * page + i < n]
    smp = np.sort(s[idx])[::-1]
    target = min(4096, max(2048, 3 * k))
    r = min(len(smp), max(1, -(-target * len(smp) // n)))
    return smp[r - 1]


def fused_topk(s, k, cap=6144):
    """The candidate path: keys >= t0 kept with their entries (any order),
    the exact top-k among them; None when the row would fall back."""
    n = len(s)
    if n <= k:
        return oracle.topk(s, k)
    t0 = -np.inf if n <= cap else sample_threshold(s, k)
    ent = np.nonzero(s >= t0)[0]
    if len(ent) < k or len(ent) > cap:
        return None
    perm = np.random.default_rng(0).permutation(len(ent))   # the candidates' order is arbitrary
    ent = ent[perm]
    order = np.lexsort((ent, -s[ent]))                      # score descending, then entry ascending
    return np.sort(ent[order[:k]]).astype(np.int32)


@pytest.mark.parametrize("n,k,kind", [
    (40000, 1024, "normal"), (66000, 1024, "normal"), (66000, 2048, "normal"),
    (50000, 512, "ties"), (30000, 1024, "signed_zero"), (60000, 1024, "rising"),
    (5000, 512, "ties"), (6000, 1024, "normal"),
])
def test_candidates_give_the_exact_top_k(n, k, kind):
    s = normal(23, "sel/%s/%d" % (kind, n), (n,))
    if kind == "ties":
        s = np.round(s * 4) / 4                  # a few hundred distinct values
    elif kind == "signed_zero":
        z = integers(23, "sel/z/%d" % n, (n,), 0, 4) == 0
        s = np.where(z, np.where(integers(23, "sel/zs/%d" % n, (n,), 0, 2) == 0, -0.0, 0.0), s)
    elif kind == "rising":
        s = s * (1.0 + 3.0 * (np.arange(n) / n) ** 4)
    want = oracle.topk(s, k)
    got = fused_topk(s, k)
    if got is None:
        pytest.skip("this row would take the stored-score path")
    assert np.array_equal(got, want)


def test_every_threshold_at_or_below_the_kth_score_is_exact():
    """Any t0 with at least k scores at or above it: the candidates hold the
    whole answer, including the lowest-index ties at the k-th score."""
    n, k = 3000, 256
    s = np.round(normal(29, "sel/any", (n,)) * 3) / 3
    want = oracle.topk(s, k)
    kth = np.sort(s)[::-1][k - 1]
    for t0 in np.unique(s[s <= kth])[-20:]:
        ent = np.nonzero(s >= t0)[0]
        assert len(ent) >= k
        order = np.lexsort((ent, -s[ent]))
        assert np.array_equal(np.sort(ent[order[:k]]), want), t0
