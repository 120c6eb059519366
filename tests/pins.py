"""Pins of the CPU oracle: checks against what the pages and the mathematics fix.

Each ``check_*`` takes an ``oracle.Oracle`` and raises AssertionError when the oracle
disagrees with a closed form, an invariant, an independent library routine, a brute
force enumeration or a hand-worked case.  ``tests/test_oracle_pins.py`` runs them on
the real oracle; ``tests/test_oracle_mutants.py`` runs them on copies of the oracle
with a planted mistake and requires every mistake to be caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bf16_bits(values) -> np.ndarray:
    """bfloat16 bit patterns of values (rounded by torch, to nearest even)."""
    t = torch.as_tensor(np.asarray(values, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def widen_bf16(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def _rng(seed):
    return np.random.default_rng(seed)


def _randn_bf16(shape, seed, scale=1.0):
    return bf16_bits(_rng(seed).standard_normal(shape) * scale)


def _close(a, b, rtol, atol=0.0, what=""):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.abs(a - b)
    lim = atol + rtol * np.abs(b)
    bad = err > lim
    assert not bad.any(), f"{what}: {int(bad.sum())} mismatches, worst {float(err.max()):.3e}"


# ---- rounding -----------------------------------------------------------------------

def check_round_bf16_vs_torch(o):
    """binary32 -> bfloat16 must equal torch's conversion (round to nearest even)."""
    rng = _rng(1)
    v = np.concatenate([
        rng.standard_normal(20000),
        rng.standard_normal(5000) * 1e30, rng.standard_normal(5000) * 1e-30,
        rng.standard_normal(5000) * 1e-39,            # binary32 subnormals
        [0.0, -0.0, 1.0, -1.0, 3.3895313892515355e38, 3.4e38, -3.4e38, np.inf, -np.inf],
    ]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = o.round_bf16(v.astype(np.float64))
    bad = got != ref
    assert not bad.any(), f"round_bf16 differs from torch at {v[bad][:5]}"
    assert (o.round_bf16(np.array([np.nan])) & 0x7FFF)[0] > 0x7F80, "NaN must stay NaN"


def _all_finite_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint32)           # +0 .. max finite
    vals = (bits << 16).view(np.float32).astype(np.float64)
    return vals, bits.astype(np.uint16)


def check_round_bf16_bruteforce(o):
    """float64 -> bfloat16 in one rounding: nearest of all bfloat16 values, ties even."""
    vals, bits = _all_finite_bf16()
    rng = _rng(2)
    k = rng.integers(1, len(vals) - 1, 20000)
    lo, hi = vals[k - 1], vals[k]
    mid = lo + (hi - lo) / 2                                # exact ties
    off = (hi - lo) * rng.uniform(-0.49, 0.49, k.shape)      # off the tie
    near = mid + off
    tiny_above = np.nextafter(mid, np.inf)
    tiny_below = np.nextafter(mid, -np.inf)
    for v in (mid, near, tiny_above, tiny_below):
        got = o.round_bf16(v)
        j = np.searchsorted(vals, v)                        # vals[j-1] < v <= vals[j]
        a, b = vals[j - 1], vals[j]
        da, db = v - a, b - v
        want = np.where(da < db, bits[j - 1], np.where(db < da, bits[j],
                        np.where(bits[j - 1] % 2 == 0, bits[j - 1], bits[j])))
        assert (got == want).all(), "round_bf16 is not nearest-even"
        assert (o.round_bf16(-v) == (want | 0x8000)).all(), "round_bf16 sign handling"


# ---- add_rms_norm: h ------------------------------------------------------------------

def check_h_exact(o):
    """h = binary32(x) + binary32(r), rounded once to the I/O type (bit exact)."""
    x = _randn_bf16((37, 96), 3)
    r = _randn_bf16((37, 96), 4, scale=3.0)
    _, h = o.add_rms_norm(x, r, None, 1e-5)
    s = (widen_bf16(x).astype(np.float32) + widen_bf16(r).astype(np.float32))
    want = torch.from_numpy(s).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (h == want).all(), "bf16 h is not RNE(x + r)"
    xf = _rng(5).standard_normal((9, 33)).astype(np.float32)
    rf = _rng(6).standard_normal((9, 33)).astype(np.float32)
    _, hf = o.add_rms_norm(xf, rf, None, 1e-5)
    assert (hf == xf + rf).all(), "f32 h is not x + r"


def check_add_rms_is_rms_of_h(o):
    """AddRmsNorm is RmsNorm of the returned (rounded) h."""
    x = _randn_bf16((21, 64), 7)
    r = _randn_bf16((21, 64), 8)
    w = bf16_bits(_rng(9).uniform(0.5, 1.5, 64))
    y, h = o.add_rms_norm(x, r, w, 1e-5)
    _close(y, o.rms_norm(h, w, 1e-5), 1e-15, what="add_rms_norm vs rms_norm(h)")


# ---- all-reduce + add_rms_norm --------------------------------------------------------

def _bf16_round_exact(v: float) -> float:
    """bfloat16 nearest-even of a double in one rounding (Python's round() ties to even
    on the exactly representable half-way value); normal range only."""
    if v == 0.0:
        return 0.0
    m, e = math.frexp(v)                 # v = m 2^e, 0.5 <= |m| < 1
    q = round(math.ldexp(m, 8))          # 8 significant bits
    return math.ldexp(q, e - 8)


def check_allreduce_rounds_exact_sum_once(o):
    """x = the sum of the partials (in double, exact here) rounded once: 1 + 2^-8 + 2^-30
    is above the bf16 tie 1 + 2^-8 and rounds up, and 1 + 2^-24 + 2^-40 above the binary32
    tie; binary32 accumulation would drop the last term and round both down to 1."""
    parts = [bf16_bits([[1.0, 3.0]]), bf16_bits([[2.0 ** -8, 2.0 ** -7]]),
             bf16_bits([[2.0 ** -30, -2.0 ** -30]])]
    r = bf16_bits([[0.0, 0.0]])
    _, _, x = o.allreduce_add_rms_norm(parts, r, None, 1e-5)
    assert widen_bf16(x).tolist() == [[1.0 + 2.0 ** -7, 3.0]], widen_bf16(x).tolist()
    pf = [np.array([[1.0]], np.float32), np.array([[2.0 ** -24]], np.float32),
          np.array([[2.0 ** -40]], np.float32)]     # exact in double, above the f32 tie
    _, _, xf = o.allreduce_add_rms_norm(pf, np.zeros((1, 1), np.float32), None, 1e-5)
    assert float(xf[0, 0]) == 1.0 + 2.0 ** -23, float(xf[0, 0])
    ps = [_randn_bf16((13, 40), 42 + i, scale=4.0 ** i) for i in range(5)]
    _, _, x = o.allreduce_add_rms_norm(ps, _randn_bf16((13, 40), 50), None, 1e-5)
    exact = sum(widen_bf16(p) for p in ps)          # exact: 8-bit significands, 10 binades
    want = np.vectorize(_bf16_round_exact)(exact)
    assert (widen_bf16(x) == want).all(), "x is not the exact sum rounded once"


def check_allreduce_order_and_cancellation(o):
    """The sum does not depend on the order of the parts (exact for bf16 data); parts
    that cancel leave x = the remaining part, h = RNE(x + r) and y = RmsNorm(h)."""
    ps = [_randn_bf16((11, 64), 60 + i) for i in range(4)]
    r = _randn_bf16((11, 64), 65)
    w = bf16_bits(_rng(66).uniform(0.5, 1.5, 64))
    y1, h1, x1 = o.allreduce_add_rms_norm(ps, r, w, 1e-5)
    y2, h2, x2 = o.allreduce_add_rms_norm(ps[::-1], r, w, 1e-5)
    assert (x1 == x2).all() and (h1 == h2).all() and (y1 == y2).all()
    p = ps[0]
    neg = p ^ np.uint16(0x8000)                      # -p exactly
    y, h, x = o.allreduce_add_rms_norm([p, neg, ps[1]], r, w, 1e-5)
    assert (x == ps[1]).all(), "p + (-p) + q must be q"
    s = widen_bf16(ps[1]).astype(np.float32) + widen_bf16(r).astype(np.float32)
    assert (h == bf16_bits(s)).all(), "h must be RNE(x + r)"
    hd = widen_bf16(h)
    want = hd / np.sqrt((hd * hd).mean(axis=1, keepdims=True) + 1e-5) * widen_bf16(w)
    _close(y, want, 1e-13, what="y = RmsNorm(h) * w")


def check_allreduce_hand_case(o):
    """parts [1, 2] and [3, 4], r = [0.5, 0.5]: x = [4, 6], h = [4.5, 6.5],
    y = h / sqrt((4.5^2 + 6.5^2) / 2 + eps); one part alone is add_rms_norm itself."""
    y, h, x = o.allreduce_add_rms_norm([bf16_bits([[1.0, 2.0]]), bf16_bits([[3.0, 4.0]])],
                                       bf16_bits([[0.5, 0.5]]), None, 1e-5)
    assert widen_bf16(x).tolist() == [[4.0, 6.0]] and widen_bf16(h).tolist() == [[4.5, 6.5]]
    den = math.sqrt((4.5 ** 2 + 6.5 ** 2) / 2 + float(np.float32(1e-5)))   # eps is binary32
    _close(y, [[4.5 / den, 6.5 / den]], 1e-15, what="hand case")
    p = _randn_bf16((7, 48), 70)
    r = _randn_bf16((7, 48), 71)
    y1, h1, x1 = o.allreduce_add_rms_norm([p], r, None, 1e-6)
    y2, h2 = o.add_rms_norm(p, r, None, 1e-6)
    assert (x1 == p).all() and (h1 == h2).all() and (y1 == y2).all()


# ---- Llama 3 frequency scaling (reading of the pages' four parameters) ----------------

def check_llama3_freqs_regions(o):
    """factor 1 changes nothing; wavelengths below orig/high keep theta exactly, those above
    orig/low get exactly theta/factor, the band between lies strictly between the two; the
    scaled frequencies fall strictly with i (the blend joins both ends continuously)."""
    dims, base = 128, 500000.0
    theta = np.array([base ** (-2.0 * i / dims) for i in range(dims // 2)])
    # (1 - s) theta + s theta rounds to within an ulp or two of theta in the band
    _close(o.llama3_freqs(dims, base, 1.0, 1.0, 4.0, 8192.0), theta, 1e-15, what="factor 1")
    for factor, low, high, orig in ((32.0, 1.0, 4.0, 8192.0), (8.0, 2.0, 16.0, 4096.0)):
        f = o.llama3_freqs(dims, base, factor, low, high, orig)
        lam = 2 * math.pi / theta
        hi, lo = lam < orig / high, lam > orig / low
        mid = ~(hi | lo)
        assert (f[hi] == theta[hi]).all(), "high frequencies must be unchanged"
        assert (f[lo] == theta[lo] / factor).all(), "low frequencies must be divided by factor"
        assert hi.any() and lo.any() and mid.any()
        assert ((f[mid] < theta[mid]) & (f[mid] > theta[mid] / factor)).all()
        assert (np.diff(f) < 0).all(), "scaled frequencies must fall strictly with i"


def check_llama3_freqs_hand_case(o):
    """dims 4, base 16: theta = [1, 1/4], wavelengths [2 pi, 8 pi]; orig 16 pi, low 1,
    high 4: thresholds 4 pi and 16 pi, so theta_0 stays and theta_1 sits in the band at
    orig / wavelength = 2, s = 1/3: (2/3)(1/4)/8 + (1/3)(1/4) = 5/48 with factor 8."""
    f = o.llama3_freqs(4, 16.0, 8.0, 1.0, 4.0, 16 * math.pi)
    assert f[0] == 1.0
    assert abs(f[1] - 5.0 / 48.0) < 1e-15, f[1]


# ---- YaRN frequency scaling (reading: the published method, in its own notation) --------

def check_yarn_freqs_regions(o):
    """s = 1 changes nothing and gives temperature 1; pairs turning more than beta times over
    the original context keep theta exactly, those turning fewer than alpha times get exactly
    theta / s, those between lie strictly between; the frequencies fall strictly with d."""
    dims, base = 128, 10000.0
    theta = np.array([base ** (-2.0 * d / dims) for d in range(dims // 2)])
    f, m = o.yarn_freqs(dims, base, 1.0, 4096.0, 1.0, 32.0)
    _close(f, theta, 1e-15, what="s = 1")
    assert m == 1.0
    for s, L, alpha, beta in ((16.0, 4096.0, 1.0, 32.0), (4.0, 2048.0, 2.0, 8.0)):
        f, _ = o.yarn_freqs(dims, base, s, L, alpha, beta)
        turns = L * theta / (2 * math.pi)
        keep, interp = turns > beta, turns < alpha
        mid = ~(keep | interp)
        assert keep.any() and interp.any() and mid.any()
        assert (f[keep] == theta[keep]).all(), "fast pairs must keep their frequency"
        assert (f[interp] == theta[interp] / s).all(), "slow pairs must be divided by s"
        assert ((f[mid] < theta[mid]) & (f[mid] > theta[mid] / s)).all()
        assert (np.diff(f) < 0).all(), "scaled frequencies must fall strictly with d"


def check_yarn_freqs_hand_case(o):
    """dims 8, base 10^4: theta = 1, 0.1, 0.01, 0.001; over L = 4096 the pairs turn
    4096 theta / (2 pi) = 651.90, 65.190, 6.518986, 0.65190 times.  With alpha 1, beta 32,
    s 4: the first two keep theta, the last gets 0.001 / 4, and the third has
    gamma = 5.518986469 / 31 = 0.1780318216, so 0.01 (0.1780318216 + 0.8219681784 / 4)
    = 0.003835238662.  Temperature 0.1 ln 4 + 1 = 1.138629436."""
    f, m = o.yarn_freqs(8, 10000.0, 4.0, 4096.0, 1.0, 32.0)
    assert f[0] == 1.0 and abs(f[1] - 0.1) < 1e-17
    assert abs(f[2] / 0.003835238662 - 1) < 1e-9, f[2]
    assert abs(f[3] - 0.00025) < 1e-19, f[3]
    assert abs(m - 1.138629436) < 1e-9, m


def check_yarn_ramp_is_the_llama3_rule(o):
    """The two readings, written separately, agree where they should: Llama 3's rule with
    low / high frequency factors (alpha, beta) and original context L is YaRN's ramp
    with those bounds (only the temperature differs)."""
    for dims, base, s, L, alpha, beta in ((128, 500000.0, 32.0, 8192.0, 1.0, 4.0),
                                          (64, 10000.0, 8.0, 4096.0, 1.0, 32.0)):
        f, _ = o.yarn_freqs(dims, base, s, L, alpha, beta)
        _close(f, o.llama3_freqs(dims, base, s, alpha, beta, L), 1e-14, what="YaRN vs Llama 3")


# ---- SuScaled (LongRoPE) frequency scaling (reading: the published method) ---------------

def check_suscaled_identity_and_selection(o):
    """Factors of 1 leave the base frequencies exactly, and a maximum context within the
    original one gives attention factor 1; the short factors serve sequences up to the
    original context L, the long ones from L + 1 on; each pair's frequency is divided by
    its own factor (the ratio of the long to the short result is short / long, pair by pair)."""
    dims, base = 64, 10000.0
    half = dims // 2
    theta = np.array([base ** (-2.0 * i / dims) for i in range(half)])
    ones = np.ones(half)
    f, m = o.suscaled_freqs(dims, base, ones, ones, 100000.0, 4096.0, 4096.0)
    _close(f, theta, 1e-15, what="factors 1")
    assert m == 1.0
    rng = _rng(21)
    short, long_ = rng.uniform(1.0, 1.5, half), rng.uniform(1.0, 40.0, half)
    fs, ms = o.suscaled_freqs(dims, base, short, long_, 4096.0, 131072.0, 4096.0)
    fl, ml = o.suscaled_freqs(dims, base, short, long_, 4097.0, 131072.0, 4096.0)
    _close(fs, theta / short, 1e-15, what="short factors at seq_len = L")
    _close(fl, theta / long_, 1e-15, what="long factors at seq_len = L + 1")
    _close(fl / fs, short / long_, 1e-14, what="per-pair ratio")
    assert ms == ml > 1.0, "the attention factor depends on the contexts, not on seq_len"


def check_suscaled_hand_case(o):
    """dims 4, base 10^4: theta = (1, 0.01).  Short factors (1, 2) give (1, 0.005); long
    factors (4, 8) give (0.25, 0.00125).  L = 4096 = 2^12 extended to L' = 131072 = 2^17:
    s = 32, ln s / ln L = 5/12, attention factor sqrt(17/12) = 1.190238071."""
    f, m = o.suscaled_freqs(4, 10000.0, [1.0, 2.0], [4.0, 8.0], 1000.0, 131072.0, 4096.0)
    assert f[0] == 1.0 and abs(f[1] - 0.005) < 1e-18, f
    f, m2 = o.suscaled_freqs(4, 10000.0, [1.0, 2.0], [4.0, 8.0], 8192.0, 131072.0, 4096.0)
    assert f[0] == 0.25 and abs(f[1] - 0.00125) < 1e-18, f
    assert m == m2 and abs(m - math.sqrt(17.0 / 12.0)) < 1e-15, m
    assert abs(m - 1.190238071) < 1e-9


# ---- rms_norm -------------------------------------------------------------------------

def check_rms_constant_rows(o):
    """A constant row c gives c*w/sqrt(c^2 + eps); a +-1 row gives +-w/sqrt(1 + eps)."""
    D = 48
    w = bf16_bits(_rng(10).uniform(0.5, 1.5, D))
    wv = widen_bf16(w)
    cs = widen_bf16(bf16_bits([0.75, -3.0, 1e-3, 250.0]))
    x = bf16_bits(np.repeat(cs[:, None], D, axis=1))
    eps = np.float32(1e-5)
    y = o.rms_norm(x, w, float(eps))
    want = cs[:, None] * wv[None, :] / np.sqrt(cs[:, None] ** 2 + float(eps))
    _close(y, want, 1e-14, what="constant rows")
    sgn = np.where(_rng(11).random((5, D)) < 0.5, -1.0, 1.0)
    y2 = o.rms_norm(bf16_bits(sgn), w, float(eps))
    _close(y2, sgn * wv / math.sqrt(1 + float(eps)), 1e-14, what="+-1 rows")


def check_rms_mean_square_invariant(o):
    """With w = 1 the output has mean square ms / (ms + eps)."""
    x = _randn_bf16((40, 128), 12, scale=0.05)
    eps = float(np.float32(1e-3))
    y = o.rms_norm(x, None, eps)
    ms = (widen_bf16(x) ** 2).mean(axis=1)
    _close((y ** 2).mean(axis=1), ms / (ms + eps), 1e-12, what="mean square")


def check_rms_scaling(o):
    """rms(c x, eps) == rms(x, eps / c^2) for c a power of two (exact rescaling)."""
    x = _randn_bf16((16, 80), 13)
    w = bf16_bits(_rng(14).uniform(0.5, 1.5, 80))
    for c in (8.0, 2.0 ** -5):
        xs = bf16_bits(widen_bf16(x) * c)
        eps = float(np.float32(1e-4))
        _close(o.rms_norm(xs, w, eps), o.rms_norm(x, w, float(np.float32(eps / c ** 2))),
               1e-14, what=f"scaling c={c}")
        _close(o.rms_norm(xs, w, 0.0), o.rms_norm(x, w, 0.0), 1e-14, what="scale invariance")


def check_rms_vs_torch(o):
    """Agreement with torch.nn.functional.rms_norm in float64 on the CPU."""
    for dt in ("bf16", "f32"):
        raw = _rng(15).standard_normal((33, 200)) * 2
        wr = _rng(16).uniform(0.5, 1.5, 200)
        if dt == "bf16":
            x, w = bf16_bits(raw), bf16_bits(wr)
            xv, wv = widen_bf16(x), widen_bf16(w)
        else:
            x, w = raw.astype(np.float32), wr.astype(np.float32)
            xv, wv = x.astype(np.float64), w.astype(np.float64)
        eps = float(np.float32(1e-6))
        ref = F.rms_norm(torch.from_numpy(xv), (200,), torch.from_numpy(wv), eps).numpy()
        _close(o.rms_norm(x, w, eps), ref, 1e-12, what=f"rms_norm vs torch ({dt})")


# ---- layer_norm -----------------------------------------------------------------------

def check_layer_norm_moments(o):
    """With w = 1, b = 0: zero mean and variance var / (var + eps)."""
    x = bf16_bits(_rng(17).standard_normal((30, 256)) * 2 + 0.5)
    eps = float(np.float32(1e-2))
    y = o.layer_norm(x, None, None, eps)
    xv = widen_bf16(x)
    var = xv.var(axis=1)
    assert (np.abs(y.mean(axis=1)) <= 1e-12 * np.abs(y).max(axis=1)).all(), "mean(y) != 0"
    _close(y.var(axis=1), var / (var + eps), 1e-10, what="var(y)")


def check_layer_norm_translation(o):
    """LayerNorm ignores a constant shift of the row (shift exact in binary32)."""
    x = _rng(18).integers(-100, 100, (12, 64)).astype(np.float32)
    w = _rng(19).uniform(0.5, 1.5, 64).astype(np.float32)
    b = _rng(20).uniform(-1, 1, 64).astype(np.float32)
    eps = float(np.float32(1e-5))
    _close(o.layer_norm(x + np.float32(1024), w, b, eps), o.layer_norm(x, w, b, eps), 1e-13,
           atol=1e-13, what="translation")


def check_layer_norm_zero_weight(o):
    """w = 0 gives y = b exactly."""
    x = _randn_bf16((6, 40), 21)
    b = bf16_bits(_rng(22).standard_normal(40) * 0.1)
    y = o.layer_norm(x, bf16_bits(np.zeros(40)), b, 1e-5)
    assert (y == widen_bf16(b)[None, :]).all(), "w = 0 must give b"


def check_layer_norm_vs_torch(o):
    """Agreement with torch.nn.functional.layer_norm in float64 on the CPU."""
    x = bf16_bits(_rng(23).standard_normal((25, 300)) * 2 + 0.5)
    w = bf16_bits(_rng(24).uniform(0.5, 1.5, 300))
    b = bf16_bits(_rng(25).standard_normal(300) * 0.1)
    eps = float(np.float32(1e-5))
    ref = F.layer_norm(torch.from_numpy(widen_bf16(x)), (300,), torch.from_numpy(widen_bf16(w)),
                       torch.from_numpy(widen_bf16(b)), eps).numpy()
    _close(o.layer_norm(x, w, b, eps), ref, 1e-12, atol=1e-13, what="layer_norm vs torch")


# ---- rope -------------------------------------------------------------------------------

def _pairs(D, dims, trad):
    half = dims // 2
    return [(2 * i, 2 * i + 1) if trad else (i, i + half) for i in range(half)]


def check_rope_norm_and_passthrough(o):
    """Each pair keeps its norm; features past dims are unchanged."""
    x = _rng(26).standard_normal((3 * 7, 40))
    for trad in (0, 1):
        y = o.rope_f64(x, 7, 24, trad, 10000.0, 1.0, 11)
        for p, q in _pairs(40, 24, trad):
            _close(y[:, p] ** 2 + y[:, q] ** 2, x[:, p] ** 2 + x[:, q] ** 2, 1e-12,
                   what="pair norm")
        assert (y[:, 24:] == x[:, 24:]).all(), "features past dims must pass through"


def check_rope_inverse(o):
    """forward = false undoes forward = true."""
    x = _rng(27).standard_normal((2 * 9, 32))
    for trad in (0, 1):
        y = o.rope_f64(x, 9, 32, trad, 500.0, 0.75, 4096, forward=True)
        _close(o.rope_f64(y, 9, 32, trad, 500.0, 0.75, 4096, forward=False), x, 1e-11,
               atol=1e-12, what="inverse")


def check_rope_position_zero(o):
    """Position 0 is the identity."""
    x = _rng(28).standard_normal((5, 16))
    for trad in (0, 1):
        assert (o.rope_f64(x, 1, 16, trad, 10000.0, 1.0, 0) == x).all(), "pos 0 must be identity"


def check_rope_shift(o):
    """(offset = o, l) is the same position as (offset = 0, l + o)."""
    x = _rng(29).standard_normal((8, 16))
    a = o.rope_f64(x, 8, 16, 0, 10000.0, 1.0, 5)
    padded = np.concatenate([np.zeros((5, 16)), x])
    b = o.rope_f64(padded, 13, 16, 0, 10000.0, 1.0, 0)[5:]
    _close(a, b, 1e-15, what="offset shift")
    # row k of a [B, H, L, D] batch is at l = k mod L
    stacked = np.concatenate([x, x])
    c = o.rope_f64(stacked, 8, 16, 0, 10000.0, 1.0, 5)
    _close(c[8:], a, 1e-15, what="l = k mod L")


def check_rope_pair_angles(o):
    """Pair i turns by pos * scale * base^(-2i/dims): theta_0 = 1, counter-clockwise."""
    base, scale, pos = 100.0, 0.25, 3
    for (dims, D), trad in [((16, 16), 0), ((16, 16), 1), ((8, 20), 0), ((8, 20), 1)]:
        rows = []
        for p, q in _pairs(D, dims, trad):
            e = np.zeros(D)
            e[p] = 1.0
            rows.append(e)
        y = o.rope_f64(np.array(rows), 1, dims, trad, base, scale, pos)
        for i, (p, q) in enumerate(_pairs(D, dims, trad)):
            ang = pos * scale * base ** (-2.0 * i / dims)
            _close([y[i, p], y[i, q]], [math.cos(ang), math.sin(ang)], 1e-14, atol=1e-15,
                   what=f"angle of pair {i}")
    # pair 0 turns by exactly pos * scale whatever the base
    e = np.zeros((1, 4))
    e[0, 0] = 1.0
    y = o.rope_f64(e, 1, 4, 0, 1234.5, 0.5, 7)
    _close(y[0, [0, 2]], [math.cos(3.5), math.sin(3.5)], 1e-15, atol=1e-16, what="theta_0 = 1")


def check_rope_traditional_is_permuted_halves(o):
    """Traditional pairs equal halves pairs conjugated by the de-interleave permutation."""
    D, dims = 20, 12
    x = _rng(30).standard_normal((6, D))
    perm = np.concatenate([np.arange(0, dims, 2), np.arange(1, dims, 2), np.arange(dims, D)])
    yt = o.rope_f64(x, 3, dims, 1, 10000.0, 1.0, 2)
    yh = o.rope_f64(x[:, perm], 3, dims, 0, 10000.0, 1.0, 2)
    back = np.empty_like(yh)
    back[:, perm] = yh
    _close(yt, back, 1e-15, what="traditional vs halves")


def check_rope_complex(o):
    """Rotation written as complex multiplication (n_p + i n_q) * exp(i phi)."""
    D, dims, L = 32, 32, 5
    x = _rng(31).standard_normal((2 * L, D))
    half = dims // 2
    y = o.rope_f64(x, L, dims, 0, 10000.0, 1.0, 100)
    pos = 100 + (np.arange(2 * L) % L)
    phi = pos[:, None] * (10000.0 ** (-np.arange(half) * 2.0 / dims))[None, :]
    z = (x[:, :half] + 1j * x[:, half:dims]) * np.exp(1j * phi)
    _close(y[:, :half], z.real, 1e-12, atol=1e-12, what="complex real")
    _close(y[:, half:dims], z.imag, 1e-12, atol=1e-12, what="complex imag")


def check_norm_rope_composition(o):
    """NormRope = Rope(RmsNorm(x, w)); normalize = 0 is Rope alone."""
    Bsz, H, L, D, dims = 2, 3, 5, 48, 32
    x = _randn_bf16((Bsz * H * L, D), 32)
    w = bf16_bits(_rng(33).uniform(0.5, 1.5, D))
    eps = float(np.float32(1e-6))
    for trad in (0, 1):
        y = o.norm_rope(x, w, L, dims, trad, 10000.0, 1.0, 4096, 1, eps)
        want = o.rope_f64(o.rms_norm(x, w, eps), L, dims, trad, 10000.0, 1.0, 4096)
        _close(y, want, 1e-15, what="norm_rope composition")
        y0 = o.norm_rope(x, w, L, dims, trad, 10000.0, 1.0, 7, 0, eps)
        _close(y0, o.rope_f64(widen_bf16(x), L, dims, trad, 10000.0, 1.0, 7), 1e-15,
               what="normalize = 0")


def check_rope_ex_matches_rope(o):
    """The general entry with default settings equals NormRope / Rope."""
    Bsz, H, L, D, dims = 2, 2, 6, 24, 16
    x = _randn_bf16((Bsz * H * L, D), 36)
    w = bf16_bits(_rng(37).uniform(0.5, 1.5, D))
    for trad in (0, 1):
        for norm in (0, 1):
            a = o.norm_rope(x, w, L, dims, trad, 500.0, 0.5, 9, norm, 1e-6)
            b = o.rope_ex(x, w, L, dims, trad, 500.0, 0.5, 9, norm, 1e-6)
            assert (a == b).all(), "rope_ex default path differs"


def check_rope_freqs(o):
    """freqs replace base^(-2i/dims): the standard frequencies reproduce Rope, zero
    frequencies leave the row unrotated, and a hand-picked quarter turn lands exactly."""
    L, D, dims = 5, 8, 8
    x = _randn_bf16((2 * L, D), 38)
    std = 100.0 ** (-np.arange(dims // 2) * 2.0 / dims)
    a = o.rope_ex(x, None, L, dims, 0, 100.0, 1.0, 3, 0, 0.0, freqs=std)
    b = o.norm_rope(x, None, L, dims, 0, 100.0, 1.0, 3, 0, 0.0)
    _close(a, b, 1e-14, atol=1e-15, what="freqs = standard")
    z = o.rope_ex(x, None, L, dims, 1, 100.0, 1.0, 3, 0, 0.0, freqs=np.zeros(dims // 2))
    assert (z == widen_bf16(x)).all(), "zero frequencies must not rotate"
    e = bf16_bits([[1.0, 0.0, 0.0, 0.0]])
    q = o.rope_ex(e, None, 1, 4, 0, 10000.0, 1.0, 1, 0, 0.0, freqs=[math.pi / 2, 0.0])
    _close(q[0], [math.cos(math.pi / 2), 0.0, 1.0, 0.0], 0, atol=1e-15, what="quarter turn")


def check_rope_ex_inverse(o):
    """forward = false undoes forward = true on the general path (no normalisation)."""
    L, D, dims = 4, 16, 12
    xf = _rng(39).standard_normal((3 * L, D)).astype(np.float32)
    for trad in (0, 1):
        y = o.rope_ex(xf, None, L, dims, trad, 1000.0, 2.0, 77, 0, 0.0, forward=True)
        back = o.rope_ex(y.astype(np.float32), None, L, dims, trad, 1000.0, 2.0, 77, 0, 0.0,
                         forward=False)
        _close(back, xf, 1e-5, atol=1e-6, what="inverse on rope_ex")


def check_rope_cache_placement(o):
    """Cache form: row (bh, l) lands at cache row (bh, offset + l); other rows untouched."""
    Bsz, H, L, D, dims, y_len, off = 1, 3, 4, 8, 8, 11, 5
    x = _randn_bf16((Bsz * H * L, D), 40)
    cache = np.full((Bsz * H * y_len, D), 7.25)
    o.rope_ex(x, None, L, dims, 0, 10000.0, 1.0, off, 1, 1e-6, y=cache, y_len=y_len)
    plain = o.norm_rope(x, None, L, dims, 0, 10000.0, 1.0, off, 1, 1e-6)
    for bh in range(Bsz * H):
        for r in range(y_len):
            got = cache[bh * y_len + r]
            if off <= r < off + L:
                assert (got == plain[bh * L + r - off]).all(), "cache row misplaced"
            else:
                assert (got == 7.25).all(), "a cache row outside [offset, offset+L) changed"


# ---- backward (vector-Jacobian products) ---------------------------------------------

def _fd_grad(f, v, h):
    """Central differences of the scalar f at v (float32 array on a dyadic grid), one
    coordinate at a time; v + h and v - h are exact in float32."""
    out = np.zeros(v.size)
    flat = v.reshape(-1)
    for i in range(flat.size):
        up, dn = flat.copy(), flat.copy()
        up[i] += np.float32(h)
        dn[i] -= np.float32(h)
        out[i] = (f(up.reshape(v.shape)) - f(dn.reshape(v.shape))) / (2 * h)
    return out.reshape(v.shape)


def _grid(shape, seed, lo=-2.0, hi=2.0):
    return (np.round(_rng(seed).uniform(lo, hi, shape) * 64) / 64).astype(np.float32)


def check_rms_norm_vjp_finite_differences(o):
    """dx and dw match central differences of the oracle's own RmsNorm."""
    x, g = _grid((3, 6), 41), _grid((3, 6), 42)
    w = _grid((6,), 43, 0.5, 1.5)
    eps = float(np.float32(1e-3))
    dx, dw, _, _ = o.rms_norm_vjp(x, w, g, eps)
    loss = lambda xx, ww: float((o.rms_norm(xx, ww, eps) * g).sum())  # noqa: E731
    _close(dx, _fd_grad(lambda xx: loss(xx, w), x, 2.0 ** -10), 1e-5, atol=1e-6, what="rms dx")
    _close(dw, _fd_grad(lambda ww: loss(x, ww), w, 2.0 ** -10), 1e-5, atol=1e-6, what="rms dw")


def check_layer_norm_vjp_finite_differences(o):
    """dx, dw and db match central differences of the oracle's own LayerNorm."""
    x, g = _grid((3, 6), 44), _grid((3, 6), 45)
    w = _grid((6,), 46, 0.5, 1.5)
    b = _grid((6,), 47, -0.5, 0.5)
    eps = float(np.float32(1e-3))
    dx, dw, db, _, _, _ = o.layer_norm_vjp(x, w, g, eps)
    loss = lambda xx, ww, bb: float((o.layer_norm(xx, ww, bb, eps) * g).sum())  # noqa: E731
    _close(dx, _fd_grad(lambda xx: loss(xx, w, b), x, 2.0 ** -10), 1e-5, atol=1e-6, what="ln dx")
    _close(dw, _fd_grad(lambda ww: loss(x, ww, b), w, 2.0 ** -10), 1e-5, atol=1e-6, what="ln dw")
    _close(db, _fd_grad(lambda bb: loss(x, w, bb), b, 2.0 ** -10), 1e-5, atol=1e-6, what="ln db")


def check_vjp_invariances(o):
    """eps = 0: RmsNorm is scale invariant (sum x dx = 0); LayerNorm is shift and scale
    invariant (sum dx = 0, sum (x - mean) dx = 0); db is the column sum of g."""
    x = _randn_bf16((7, 40), 48)
    g = _randn_bf16((7, 40), 49)
    w = bf16_bits(_rng(50).uniform(0.5, 1.5, 40))
    xv = widen_bf16(x)
    dx, _, _, _ = o.rms_norm_vjp(x, w, g, 0.0)
    scale = np.abs(dx).max(axis=1) * np.abs(xv).max(axis=1) * 40
    assert (np.abs((xv * dx).sum(axis=1)) <= 1e-13 * scale).all(), "rms: x . dx != 0"
    dx, _, db, _, _, _ = o.layer_norm_vjp(x, w, g, 0.0)
    s = np.abs(dx).max(axis=1) * 40
    assert (np.abs(dx.sum(axis=1)) <= 1e-13 * s).all(), "layer: sum dx != 0"
    xc = xv - xv.mean(axis=1, keepdims=True)
    assert (np.abs((xc * dx).sum(axis=1)) <= 1e-12 * s * np.abs(xc).max()).all(), \
        "layer: (x - mean) . dx != 0"
    _close(db, widen_bf16(g).sum(axis=0), 1e-14, atol=1e-14, what="db")


def check_vjp_without_weight(o):
    """w = None is w = 1 and has no gradient of its own."""
    x, g = _randn_bf16((5, 24), 51), _randn_bf16((5, 24), 52)
    ones = bf16_bits(np.ones(24))
    a = o.rms_norm_vjp(x, None, g, 1e-5)
    b = o.rms_norm_vjp(x, ones, g, 1e-5)
    assert a[1] is None and (a[0] == b[0]).all(), "rms vjp with w = None"
    a = o.layer_norm_vjp(x, None, g, 1e-5)
    b = o.layer_norm_vjp(x, ones, g, 1e-5)
    assert a[1] is None and (a[0] == b[0]).all() and (a[2] == b[2]).all(), "layer vjp w = None"


# ---- hand-worked cases -----------------------------------------------------------------

_MATH = {k: getattr(math, k) for k in ("sqrt", "cos", "sin", "pi")}


def _io_array(vals, dt):
    if vals is None:
        return None
    a = np.asarray(vals, np.float64)
    if dt == "bf16":
        b = bf16_bits(a)
        assert (widen_bf16(b) == a).all(), "hand case input not exact in bf16"
        return b
    f = a.astype(np.float32)
    assert (f.astype(np.float64) == a).all(), "hand case input not exact in f32"
    return f


def check_hand_cases(o):
    """Cases worked by hand from the definitions (tests/golden/hand_cases.json)."""
    with open(os.path.join(GOLDEN, "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        dt = c["dtype"]
        x = _io_array(c["x"], dt)
        w = _io_array(c.get("w"), dt)
        eps = c["eps"]
        want = np.array([[eval(e, {"__builtins__": {}}, _MATH) for e in row]
                         for row in c["expected"]])
        if c["op"] == "rms_norm":
            y = o.rms_norm(x, w, eps)
        elif c["op"] == "add_rms_norm":
            y, h = o.add_rms_norm(x, _io_array(c["r"], dt), w, eps)
            hv = widen_bf16(h) if dt == "bf16" else h.astype(np.float64)
            assert (hv == np.asarray(c["expected_h"])).all(), f"{c['name']}: h"
        elif c["op"] == "layer_norm":
            y = o.layer_norm(x, w, _io_array(c.get("b"), dt), eps)
        elif c["op"] == "norm_rope":
            y = o.norm_rope(x, w, c["L"], c["dims"], c["traditional"], c["base"], c["scale"],
                            c["offset"], c["normalize"], eps)
        else:
            raise AssertionError(f"unknown op {c['op']}")
        _close(y, want, 1e-14, atol=1e-15, what=c["name"])


def check_minivllm_example(o):
    """The residual example of the miniVLLM Layers page (shapes only on the page)."""
    with open(os.path.join(GOLDEN, "minivllm_example.json")) as f:
        ex = json.load(f)
    shape = ex["shape"]
    rows, D = int(np.prod(shape[:-1])), shape[-1]
    x = _rng(34).standard_normal((rows, D)).astype(np.float32)
    r = _rng(35).standard_normal((rows, D)).astype(np.float32)
    w = np.ones(D, np.float32)
    eps = float(np.float32(ex["eps"]))
    y, h = o.add_rms_norm(x, r, w, eps)
    assert (h == x + r).all(), "updated residual must be x + residual"
    ms = (h.astype(np.float64) ** 2).mean(axis=1)
    _close((y ** 2).mean(axis=1), ms / (ms + eps), 1e-12, what="example mean square")


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
