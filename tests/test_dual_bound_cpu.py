"""The dual-means error bound, checked on the host.

The refining top-k treats a block as decided when its bf16 score lies more than
e = scale (|q|_2 (1 + 2^-10) + 2^-59) rho from a threshold, rho being the row's stored
radius (1 + 2^-12)|m - bf16(m)|_2 + 2^-18 |m|_2 + 2^-59, all rounded up.  That is sound
only if e bounds the gap between the two fp32 scores the kernels compute:
* the dual scan's: lane x (16 per row) sums dims 8x..8x+7 of q * bf16(m) in one fma
  chain, then the 16 lane partials pair by xor 8, 4, 2, 1;
* the fp32 scan's (and the refinement's rescoring): lane l (32 per row) sums dims
  4l..4l+3 of q * m in one fma chain, then the 32 partials pair by xor 16, 8, 4, 2, 1;
each times the scale.  Here both are emulated in that operation order (a product and an
fma round once to fp32, through fp64 where the product is exact), on rows built to
stress the bound, and the gap must stay within e.  A control drops the 2^-18 |m|_2 term
(the fp32 rounding of the two sums): on rows whose means are exactly bf16 values the
two scores differ only by their summation orders, and that bound must fail there.
"""
import numpy as np

F32 = np.float32
SCALE = F32(1.0 / np.sqrt(np.float32(128)))


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32)


def fma(a, b, c):
    """fp32 fma: one rounding of a * b + c (the fp64 product of two fp32 values is exact;
    the fp64 sum then rounds once more, at most one fp64 ulp, far below the bound's
    slack)."""
    return f32(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def up(x64):
    """The fp32 value at or above an fp64 value (directed rounding up)."""
    y = f32(x64)
    return np.where(y.astype(np.float64) < x64, np.nextafter(y, F32(np.inf)), y)


def bf16_rne(m):
    """fp32 -> bf16 rounding to nearest even, back as fp32 (finite inputs)."""
    u = m.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (r << 16).astype(np.uint32).view(np.float32)


def xor_tree(parts):
    """Sum lane partials [..., n] by the pairing tree xor n/2, ..., 1 (fp32 adds):
    every lane ends with the same total; lane 0's is returned."""
    v = parts.copy()
    n = v.shape[-1]
    off = n // 2
    lanes = np.arange(n)
    while off >= 1:
        v = f32(v.astype(np.float64) + v[..., lanes ^ off].astype(np.float64))
        off //= 2
    return v[..., 0]


def chain(q, m, width):
    """Per-lane fma chains: lane j sums dims width*j .. width*j + width - 1, first term a
    rounded product, the rest fmas in dim order."""
    rows, d = m.shape
    qm = q.reshape(1, d // width, width)
    mm = m.reshape(rows, d // width, width)
    t = f32(qm[..., 0].astype(np.float64) * mm[..., 0].astype(np.float64))
    for c in range(1, width):
        t = fma(qm[..., c], mm[..., c], t)
    return t


def fp32_score(q, m):
    return f32(xor_tree(chain(q, m, 4)).astype(np.float64) * np.float64(SCALE))


def dual_score(q, m):
    return f32(xor_tree(chain(q, bf16_rne(m), 8)).astype(np.float64) * np.float64(SCALE))


def radius(m, rounding_term=True):
    """The stored radius as the build kernel computes it: fp32 sums of squares (lane fma
    chains over 4 dims, xor tree over 32 lanes), square roots and the combination rounded
    up."""
    d = f32(m.astype(np.float64) - bf16_rne(m).astype(np.float64))
    dd = xor_tree(_sq_chain(d))
    mm = xor_tree(_sq_chain(m))
    a = up(np.sqrt(dd.astype(np.float64)))
    a = up(a.astype(np.float64) * (1 + 2.0 ** -12))
    b = up(np.sqrt(mm.astype(np.float64)))
    b = up(b.astype(np.float64) * 2.0 ** -18) if rounding_term else np.zeros_like(b)
    return up(up(a.astype(np.float64) + b.astype(np.float64)).astype(np.float64) + 2.0 ** -59)


def _sq_chain(x):
    """Lane partials of sum x^2 as the build kernel forms them: x0*x0, then fmas."""
    rows, d = x.shape
    xx = x.reshape(rows, d // 4, 4)
    t = f32(xx[..., 0].astype(np.float64) ** 2)
    for c in range(1, 4):
        t = fma(xx[..., c], xx[..., c], t)
    return t


def err_scale(q):
    """scale (|q|_2 (1 + 2^-10) + 2^-59), |q|_2 from an fp32 sum of squares (lane fma
    chains over 4 dims, xor tree over 32 lanes), rounded up."""
    qq = xor_tree(_sq_chain(q.reshape(1, -1)))[0]
    n = up(np.sqrt(np.float64(qq)))
    n = up(up(np.float64(n) * (1 + 2.0 ** -10)).astype(np.float64) + 2.0 ** -59)
    return up(np.float64(n) * np.float64(SCALE))


def summed_query(rng, g, spread):
    """g bf16 query rows summed in row order in fp32, magnitudes spread over 2^spread."""
    q = rng.standard_normal((g, 128)) * np.exp2(rng.integers(-spread, spread + 1, (g, 128)))
    q = bf16_rne(f32(q))
    s = np.zeros(128, F32)
    for j in range(g):
        s = f32(s.astype(np.float64) + q[j].astype(np.float64))
    return s


def stress_rows(rng, n, kind):
    """Means that stress the bound.  'midpoint': just under a bf16 rounding midpoint, so the
    rounding residual is near its largest; 'exact': bf16 values (zero residual), with big
    terms of both signs so the score cancels and only the summation orders differ;
    'tiny': magnitudes near 2^-70; 'wide': exponents spread over 2^-30..2^30."""
    if kind == "midpoint":
        base = bf16_rne(f32(rng.standard_normal((n, 128))))
        ulp = f32(np.abs(base).astype(np.float64) * 2.0 ** -7)
        return f32(base.astype(np.float64) + np.sign(base) * ulp * (0.5 - 2.0 ** -9))
    if kind == "exact":
        big = rng.standard_normal((n, 128)) * np.exp2(rng.integers(0, 12, (n, 128)))
        return bf16_rne(f32(big))
    if kind == "tiny":
        return f32(rng.standard_normal((n, 128)) * 2.0 ** -70)
    if kind == "wide":
        return f32(rng.standard_normal((n, 128)) * np.exp2(rng.integers(-30, 31, (n, 128))))
    raise ValueError(kind)


def gaps(kind, seed, rounding_term=True, n=3000, g=8, spread=6):
    rng = np.random.default_rng(seed)
    q = summed_query(rng, g, spread)
    if kind == "tiny":
        q = f32(q.astype(np.float64) * 2.0 ** -70)
    m = stress_rows(rng, n, kind)
    s = fp32_score(q, m).astype(np.float64)
    st = dual_score(q, m).astype(np.float64)
    e = up(np.float64(err_scale(q)) * radius(m, rounding_term).astype(np.float64)).astype(np.float64)
    return np.abs(st - s), e


def test_helpers_match_their_definitions():
    # bf16 rounding: ties to even, and the round trip of bf16 values is exact
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9, -2.5], np.float32)
    assert list(bf16_rne(x)) == [1.0, 1.0 + 2 * 2.0 ** -7, 1.0, -2.5]
    # the xor tree sums exactly representable values exactly
    v = np.arange(32, dtype=np.float32).reshape(1, 32)
    assert xor_tree(v)[0] == 496.0
    # a product of two fp32 values is exact in fp64, so fma rounds once
    # (1 + 2^-12)^2 = 1 + 2^-11 + 2^-24: the rounded product ties to the even 1 + 2^-11
    a, c = np.float32(1 + 2.0 ** -12), np.float32(-(1 + 2.0 ** -11))
    assert fma(a, a, c) == np.float32(2.0 ** -24)
    assert f32(np.float64(a) * np.float64(a)) + c == 0.0
    # rounding up never lands below
    y = np.array([1 / 3, 2.0 ** -140, 7.0], np.float64)
    assert np.all(up(y).astype(np.float64) >= y)


def test_bound_holds_on_stress_rows():
    for kind in ("midpoint", "exact", "tiny", "wide"):
        for seed in range(3):
            gap, e = gaps(kind, seed)
            assert np.all(gap <= e), (kind, seed, float(np.max(gap / np.maximum(e, 1e-300))))


def test_bound_is_not_loose_by_orders_of_magnitude():
    # on means just under bf16 midpoints the residual term is the bound, and real gaps
    # come within a small factor of it (Cauchy-Schwarz is tight only for aligned q, d)
    gap, e = gaps("midpoint", 7)
    assert np.max(gap / e) > 1e-3


def test_control_without_the_rounding_term_fails_on_exact_rows():
    # bf16-exact means: zero residual, so only the fp32 rounding term covers the two
    # summation orders; without it the bound is the 2^-59 floor and some rows exceed it
    gap, e = gaps("exact", 11, rounding_term=False)
    assert np.any(gap > e)
    gap, e = gaps("exact", 11)
    assert np.all(gap <= e)
