"""The division-free NVFP4 code rule of the GDN fold kernel, checked in IEEE float32 on the host.

The fold re-quantises the read copy in registers ("Hybrid-model decoding has a new bottleneck", Interpretation,
fourth paragraph).  Each element's E2M1 code is the round-to-nearest-even index of the correctly rounded
quotient |x| / d_b.  The kernel avoids the division: with r = 1/d_b correctly rounded it forms q' = |x| r and
takes the code of q'(1 - 2^-19) and of q'(1 + 2^-19); where the two agree, that is the code, otherwise the
element falls back to the division.  This test replays the rule with numpy's float32 arithmetic (correctly
rounded, like the kernel's __frcp_rn and __fmul_rn) on quotients placed within a few ulps of every decision
threshold, and checks that (1) the bracket never agrees on a wrong code and (2) it falls back rarely.
"""

import numpy as np

F32 = np.float32
THRESHOLDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def e2m1_index(y):
    """Index 0..7 of {0, .5, 1, 1.5, 2, 3, 4, 6} nearest to y >= 0, ties to the even index, saturating."""
    y = np.asarray(y, dtype=F32)
    n = np.where(y < 2, np.rint(y * F32(2)), np.where(y < 4, np.rint(y) + 2, np.rint(y * F32(0.5)) + 4))
    return np.minimum(n, 7).astype(np.int64)


def _e4m3_values():
    e = np.arange(16)[:, None]
    m = np.arange(8)[None, :]
    v = np.where(e == 0, m * 2.0 ** -9, (8 + m) * 2.0 ** (e - 10)).ravel()
    return v[(v > 0) & (v <= 448)]


def _cases(rng, n_steps=48):
    """(x, d) pairs in float32: quotients near each threshold (a few ulps either side), then random ones (their
    count is returned third)."""
    sb = _e4m3_values()
    d = (rng.choice(sb, 4096) * rng.uniform(1e-6, 1e3, 4096)).astype(F32)
    d = d[d > 0]
    xs, ds = [], []
    for th in THRESHOLDS:
        for k in range(-n_steps, n_steps + 1):
            t = F32(th) * (F32(1) + F32(k) * F32(2.0 ** -24))
            x = (t * d).astype(F32)
            for dx in (-1, 0, 1):  # neighbours of the product as well
                xs.append(np.nextafter(x, np.inf) if dx > 0 else np.nextafter(x, 0) if dx < 0 else x)
                ds.append(d)
    q = rng.uniform(0, 7, d.size).astype(F32)
    xs.append((q * d).astype(F32))
    ds.append(d)
    return np.concatenate(xs).astype(F32), np.concatenate(ds).astype(F32), d.size


def test_bracketed_codes_equal_the_division_codes():
    rng = np.random.default_rng(7)
    x, d, n_rand = _cases(rng)
    with np.errstate(over="ignore", divide="ignore"):
        ref = e2m1_index(np.abs(x) / d)                   # correctly rounded float32 quotient
        r = F32(1) / d
        qp = np.abs(x) * r
        lo = e2m1_index(qp * F32(1 - 2.0 ** -19))
        hi = e2m1_index(qp * F32(1 + 2.0 ** -19))
    agree = lo == hi
    assert np.array_equal(lo[agree], ref[agree])
    # the quotients were placed on the thresholds on purpose, so some fall back; on the random tail almost none do
    assert agree.mean() > 0.2
    tail = slice(x.size - n_rand, x.size)
    assert agree[tail].mean() > 0.999


def test_index_rule_is_monotone_and_ties_to_even():
    y = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 1e9], dtype=F32)
    assert e2m1_index(y).tolist() == [0, 2, 2, 4, 4, 6, 6, 7, 7, 7]
    grid = np.sort(np.random.default_rng(1).uniform(0, 8, 100000).astype(F32))
    assert np.all(np.diff(e2m1_index(grid)) >= 0)
