"""The candidate top-k's selection rule, modelled in exact integer key arithmetic on the CPU.

The decode step's indexer keeps every score at or above a threshold tau (its candidate lists),
and the top-k selects among them: one histogram of (key - key(tau)) >> 12 over 4,096 bins (the
last open-ended), the bin of the k-th largest key from the top, every key in a higher bin
chosen, the keys of that bin ranked exactly (larger key, then lower position) when at most 64
of them, else the k-th key T found by a radix pass over the bin's low 12 bits (or 12 bits at a
time over the whole key for the open bin) and the keys equal to T taken lowest position first.
This model follows those steps (numpy, uint32 keys) and is checked against the oracle's top-k
over the whole request: the rule must be exact for any tau that leaves at least k candidates.
"""
import numpy as np
import pytest

from oracle import ls_oracle as O

BINS, SHIFT, LIST = 4096, 12, 64


def fkey(x):
    """Order-preserving uint32 key of float32 values (larger float -> larger key)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return np.where(b & 0x80000000, (~b) & 0xFFFFFFFF, b | 0x80000000).astype(np.uint64)


def kth_by_radix(vals, k, width_bits, hi):
    """The k-th largest of `vals` (non-negative ints < 2**hi) by radix passes of up to 12 bits
    from bit hi down; returns (value, how many equal to it are taken)."""
    prefix, k_rem = 0, k
    while hi > 0:
        width = min(width_bits, hi)
        shift = hi - width
        sel = vals[(vals >> hi) == prefix] if hi < 64 else vals
        digits = (sel >> shift) & ((1 << width) - 1)
        hist = np.bincount(digits.astype(np.int64), minlength=1 << width)
        above = 0
        for d in range((1 << width) - 1, -1, -1):
            if above + hist[d] >= k_rem:
                prefix = (prefix << width) | d
                k_rem -= above
                break
            above += hist[d]
        hi = shift
    return prefix, k_rem


def model_select(scores, tau, k):
    scores = np.asarray(scores, dtype=np.float32)
    keys = fkey(scores)
    tk = int(fkey(np.float32(tau)))
    cand = np.nonzero(scores >= np.float32(tau))[0]          # complete lists
    assert cand.size >= k
    ck, cp = keys[cand], cand
    d = ck - tk
    bins = np.minimum(d >> SHIFT, BINS - 1)
    hist = np.bincount(bins.astype(np.int64), minlength=BINS)
    above = 0
    for tb in range(BINS - 1, -1, -1):
        if above + hist[tb] >= k:
            break
        above += hist[tb]
    r0 = k - above
    chosen = np.zeros(scores.size, dtype=bool)
    chosen[cp[bins > tb]] = True
    inbin = bins == tb
    if inbin.sum() <= LIST:
        # exact rank inside the bin
        bk, bp = ck[inbin], cp[inbin]
        rank = np.array([np.sum((bk > bk[e]) | ((bk == bk[e]) & (bp < bp[e]))) for e in range(bk.size)])
        chosen[bp[rank < r0]] = True
        route = "list"
    else:
        if tb < BINS - 1:  # one pass over the bin's low 12 bits
            sub, R = kth_by_radix(d[inbin] & ((1 << SHIFT) - 1), r0, 12, SHIFT)
            T = tk + ((tb << SHIFT) | sub)
            route = "bin pass"
        else:              # the open bin: whole keys, 12 bits at a time
            T, R = kth_by_radix(ck, k, 12, 32)
            route = "whole key"
        chosen[cp[ck > T]] = True
        ties = np.sort(cp[ck == T])
        chosen[ties[:R]] = True
    out = np.nonzero(chosen)[0]
    assert out.size == k
    return out.astype(np.int32), route


def check(scores, tau, k):
    got, route = model_select(scores, tau, k)
    want, _ = O.topk_select(np.asarray(scores, dtype=np.float32).astype(np.float64), k)
    assert np.array_equal(got, want), route
    return route


@pytest.mark.parametrize("quantile", [0.016, 0.02, 0.03, 0.045])
def test_iid_scores_various_thresholds(quantile):
    rng = np.random.default_rng(11)
    s = rng.standard_normal(131072).astype(np.float32)
    tau = np.quantile(s, 1 - quantile).astype(np.float32)
    assert check(s, tau, 2048) == "list"


def test_threshold_exactly_at_the_kth_score():
    rng = np.random.default_rng(12)
    s = rng.standard_normal(40000).astype(np.float32)
    tau = np.sort(s)[::-1][999]                      # exactly k candidates
    check(s, tau, 1000)


def test_ties_across_the_kth_key():
    rng = np.random.default_rng(13)
    s = rng.standard_normal(131072).astype(np.float32)
    v = np.sort(s)[::-1][2000]
    s[rng.choice(s.size, 600, replace=False)] = v      # 600 equal keys around rank 2000
    tau = np.quantile(s, 0.97).astype(np.float32)
    assert check(s, tau, 2048) == "bin pass"


def test_crowded_bin_without_ties():
    # scores 1 ulp apart, 3000 of them inside one 4096-key bin just above tau
    base = np.float32(1.0)
    steps = np.arange(3000, dtype=np.uint32)
    s = (np.full(3000, base, dtype=np.float32).view(np.uint32) + steps).view(np.float32)
    rng = np.random.default_rng(14)
    s = np.concatenate([s, rng.uniform(-1, 0.5, 20000).astype(np.float32)])
    rng.shuffle(s)
    assert check(s, base, 2048) == "bin pass"


def test_open_last_bin():
    # tau far below the scores: every candidate lands in the open last bin
    rng = np.random.default_rng(15)
    s = rng.uniform(1e3, 2e3, 8000).astype(np.float32)
    assert check(s, np.float32(1e-6), 2048) == "whole key"


def test_negative_scores_and_threshold():
    rng = np.random.default_rng(16)
    s = (rng.standard_normal(50000) - 10).astype(np.float32)
    tau = np.quantile(s, 0.95).astype(np.float32)
    assert tau < 0
    check(s, tau, 2048)


def test_all_candidates_chosen():
    rng = np.random.default_rng(17)
    s = rng.standard_normal(5000).astype(np.float32)
    tau = np.sort(s)[::-1][511]
    check(s, tau, 512)
