"""A host model of the GPU top-p select's decision procedure, checked against the oracle.

The kernels do not sort: they histogram the fixed-point masses over linear buckets of the
score range, find the bucket where the cumulative mass from the top reaches ceil(p Z),
resolve that bucket either by ordering its few members or by radix digits of the fp64
order key below the bucket's common key prefix, and keep everything above the cutoff plus
the first `need` members of a final tie group in position (= id) order.  This model
follows those steps on the host and must keep exactly the set the oracle's sort-based
top-p keeps, for every score distribution below (ties, near-ties, huge ranges, one value).
It does not run the kernels; the GPU parity tests do.
"""
from __future__ import annotations

import math
import zlib

import numpy as np
import pytest

from oracle import zha_oracle as zo


def okey(s):
    b = np.asarray(s, np.float64).view(np.uint64)
    neg = (b >> np.uint64(63)).astype(bool)
    return np.where(neg, ~b, b | np.uint64(1 << 63))


def digits(s, M, Mn, nb):
    r = M - Mn
    iw = nb / r if r > 0 else 0.0
    if not math.isfinite(iw) or iw == 0.0:
        return np.full(len(s), nb - 1)
    x = (M - s) * iw
    return np.where(x < nb - 1, nb - 1 - np.floor(np.minimum(x, nb)).astype(np.int64), 0)


def boundary(mass, above, tgt):
    acc = above
    for b in range(len(mass) - 1, -1, -1):
        if acc + mass[b] >= tgt:
            return b, acc
        acc += mass[b]
    raise AssertionError("no boundary bucket")


def model_select(s, E, p, nb=2048, wd=11, members=32, k=None):
    """With k (the fixed-count selector) every candidate weighs 1 and the target is k."""
    n = len(s)
    if n == 0 or (p >= 1.0 if k is None else k >= n):
        return np.arange(n)
    Z = int(sum(int(e) for e in E))
    tgt = max(1, min(Z, math.ceil(p * Z))) if k is None else k
    d = digits(s, s.max(), s.min(), nb)
    mass = [0] * nb
    cnt = np.bincount(d, minlength=nb)
    for i in range(n):
        mass[d[i]] += int(E[i])
    d1, above = boundary(mass, 0, tgt)
    keys = okey(s)
    mem = np.nonzero(d == d1)[0]
    shift, pfx, need, cnt_t = 64, 0, 0, 0
    if cnt[d1] > 1 and cnt[d1] <= members:
        # walk the members in (key desc, position asc) order
        order = sorted(mem, key=lambda i: (-int(keys[i]), i))
        acc, last = above, order[-1]
        for i in order:
            acc += int(E[i])
            if acc >= tgt:
                last = i
                break
        pfx, shift = int(keys[last]), 0
        ties = [i for i in mem if int(keys[i]) == pfx]
        cnt_t, need = len(ties), sum(1 for i in ties if i <= last)
    elif cnt[d1] > 1:
        kmx, kmn = int(keys[mem].max()), int(keys[mem].min())
        cnt_b, mass_b = int(cnt[d1]), mass[d1]
        if kmx == kmn:
            pfx, shift = kmx, 0
        else:
            hi = (kmx ^ kmn).bit_length() - 1
            pfx = 0 if hi == 63 else kmx >> (hi + 1)
            while True:
                width = min(hi + 1, wd)
                lo = hi + 1 - width
                m2 = [0] * (1 << width)
                c2 = [0] * (1 << width)
                for i in mem:
                    k = int(keys[i])
                    if (0 if hi == 63 else k >> (hi + 1)) == pfx:
                        bkt = (k >> lo) & ((1 << width) - 1)
                        c2[bkt] += 1
                        m2[bkt] += int(E[i])
                bstar, above = boundary(m2, above, tgt)
                cnt_b, mass_b = c2[bstar], m2[bstar]
                pfx = (pfx << width) | bstar
                if cnt_b <= 1 or lo == 0:
                    shift = lo
                    break
                hi = lo - 1
        cnt_t = cnt_b
        if cnt_b <= 1:
            need = 1
        else:
            e1 = mass_b // cnt_b
            need = max(1, min(cnt_b, cnt_b if e1 == 0 else (tgt - above + e1 - 1) // e1))
    out, ties = [], 0
    partial = shift != 64 and cnt_t > 1 and need < cnt_t
    for i in range(n):
        if d[i] != d1:
            keep = d[i] > d1
        elif shift == 64:
            keep = True
        else:
            kk = int(keys[i]) >> shift
            if kk != pfx:
                keep = kk > pfx
            else:
                keep = not partial or ties < need
                ties += 1
        if keep:
            out.append(i)
    return np.array(out, dtype=np.int64)


def fixed_masses(s, S=50):
    M = float(np.max(s))
    return [int(round(math.ldexp(math.exp(v - M), S))) for v in s]


def reference(s, E, p):
    n = len(s)
    if p >= 1.0 or n == 0:
        return np.arange(n)
    Z = sum(E)
    tgt = max(1, min(Z, math.ceil(p * Z)))
    acc, out = 0, []
    for i in sorted(range(n), key=lambda i: (-s[i], i)):
        out.append(i)
        acc += E[i]
        if acc >= tgt:
            break
    return np.array(sorted(out), dtype=np.int64)


@pytest.mark.parametrize("kind", ["normal", "narrow", "quartered", "outlier", "constant", "wide_range"])
@pytest.mark.parametrize("nb,wd", [(256, 8), (2048, 11)])
def test_bucket_select_equals_sorted_cutoff(kind, nb, wd):
    rng = np.random.default_rng(zlib.crc32(f"{kind}/{nb}".encode()))
    for trial in range(60):
        n = int(rng.integers(1, 700))
        if kind == "normal":
            s = rng.normal(size=n)
        elif kind == "narrow":
            s = rng.normal(size=n) * 1e-3
        elif kind == "quartered":
            s = np.round(rng.normal(size=n) * 4) / 4          # large exact tie groups
        elif kind == "outlier":
            s = np.concatenate([rng.normal(size=n - 1) * 1e-9, [30.0]])
        elif kind == "constant":
            s = np.full(n, 1.25)
        else:
            s = rng.exponential(size=n) * rng.choice([1, -1], size=n) * 10.0 ** rng.integers(-8, 3, size=n)
        s = s.astype(np.float64)
        s[s == 0] = 0.0
        E = fixed_masses(s)
        p = float(rng.choice([0.3, 0.5, 0.9, 0.95, 0.99, 0.999, 1.0]))
        for members in (0, 32):                              # radix-only and member walk
            got = model_select(s, E, p, nb, wd, members)
            assert np.array_equal(got, reference(s, E, p)), (kind, trial, n, p, members)


def test_reference_matches_oracle_top_p_on_distinct_scores():
    """The integer-mass reference above keeps the oracle's set when no cutoff is within
    rounding of p (the oracle sums fp64 probabilities)."""
    rng = np.random.default_rng(5)
    for _ in range(40):
        s = rng.normal(size=int(rng.integers(2, 400))) * 2
        p = float(rng.choice([0.5, 0.9, 0.95]))
        sel = zo.top_p(s, np.arange(len(s), dtype=np.int64), p)
        if sel.margin < 1e-9:
            continue
        assert np.array_equal(np.sort(sel.ids), reference(s, fixed_masses(s), p))


@pytest.mark.parametrize("kind", ["normal", "quartered", "outlier", "constant", "wide_range"])
@pytest.mark.parametrize("nb,wd", [(256, 8), (2048, 11)])
def test_bucket_select_with_unit_masses_is_top_k(kind, nb, wd):
    """The fixed-count selector runs the same procedure with a mass of 1 per candidate and
    the target k: it must keep the oracle's top-k set (ties broken by position)."""
    rng = np.random.default_rng(zlib.crc32(f"{kind}/{nb}/k".encode()))
    for trial in range(60):
        n = int(rng.integers(1, 700))
        if kind == "normal":
            s = rng.normal(size=n)
        elif kind == "quartered":
            s = np.round(rng.normal(size=n) * 4) / 4
        elif kind == "outlier":
            s = np.concatenate([rng.normal(size=n - 1) * 1e-9, [30.0]])
        elif kind == "constant":
            s = np.full(n, 1.25)
        else:
            s = rng.exponential(size=n) * rng.choice([1, -1], size=n) * 10.0 ** rng.integers(-8, 3, size=n)
        s = s.astype(np.float64)
        s[s == 0] = 0.0            # one zero: the order key tells -0.0 below +0.0, a sort does not
        k = int(rng.integers(1, n + 3))
        want = zo.top_k(s, np.arange(n, dtype=np.int64), k).ids
        for members in (0, 32):
            got = model_select(s, [1] * n, None, nb, wd, members, k=k)
            assert np.array_equal(got, want), (kind, trial, n, k, members)
