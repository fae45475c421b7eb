"""Pins of the CPU oracle to facts fixed outside it: the pages' printed numbers,
closed forms, independent library routines, exact rational brute force and
algebraic identities.  CPU only."""

import json
import math
import os
import statistics
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O

F32 = np.float32


# ---------------------------------------------------------------------------
# Normal quantile (AS241)
# ---------------------------------------------------------------------------
def test_ppf_matches_two_independent_libraries():
    # statistics.NormalDist and scipy (Cephes ndtri) are separate implementations.
    nd = statistics.NormalDist()
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 4001), [1e-300, 1e-20, 1e-10, 0.02, 0.075, 0.925,
                                                            0.9677083, 0.5 + 1e-12, 1 - 1e-12]])
    for p in ps:
        got = O.norm_ppf(float(p))
        ref1 = nd.inv_cdf(float(p))
        ref2 = float(scipy.special.ndtri(p))
        tol = 4e-16 * max(1.0, abs(ref1))
        assert abs(got - ref1) <= tol + 1e-300, (p, got, ref1)
        assert abs(got - ref2) <= 1e-13 * max(1.0, abs(ref2)), (p, got, ref2)


def test_ppf_inverts_erf_cdf():
    # Phi(x) = (1 + erf(x / sqrt 2)) / 2 from the C library, a different route.
    for x in np.linspace(-6, 6, 241):
        p = 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))
        if 1e-12 < p < 1 - 1e-12:
            assert abs(O.norm_ppf(p) - x) < 1e-7 * max(1.0, abs(x)) + 1e-9
    assert O.norm_ppf(0.5) == 0.0


# ---------------------------------------------------------------------------
# NF4 level table
# ---------------------------------------------------------------------------
def test_levels_structure():
    lv = O.nf4_levels()
    assert lv.dtype == np.float32 and lv.shape == (16,)
    assert np.all(np.diff(lv) > 0)                    # 16 sorted, distinct levels
    assert lv[7] == 0.0 and np.signbit(lv[7]) == 0    # exact zero
    assert lv[0] == -1.0 and lv[15] == 1.0            # endpoints +-1
    assert np.sum(lv > 0) == 8 and np.sum(lv < 0) == 7  # 8 positive, 7 negative
    assert float(np.min(np.diff(lv))) == pytest.approx(0.0795803, abs=1e-7)


def _torch_fp32_levels():
    """The glossary snippet's construction, re-expressed in torch float32."""
    nrm = torch.distributions.Normal(0.0, 1.0)
    up = nrm.icdf(torch.linspace(0.9677083, 0.5, 9)[:-1])
    dn = -nrm.icdf(torch.linspace(0.9677083, 0.5, 8)[:-1])
    t = torch.cat([dn, torch.zeros(1), up]).sort().values
    return (t / t.max()).numpy()


def test_levels_close_to_snippet_float32_build():
    # The snippet builds the table with several float32 roundings (linspace, icdf,
    # the division by the max); the oracle rounds the exact values once.  The two
    # agree to float32 working precision (a few ulp on the small levels).
    ours = O.nf4_levels().view(np.int32).astype(np.int64)
    theirs = _torch_fp32_levels().view(np.int32).astype(np.int64)
    assert np.max(np.abs(ours - theirs)) <= 8
    assert np.sum(ours != theirs) <= 12


def _levels_from_library_ppf(ppf):
    """The snippet's construction with a library quantile in float64, each level
    rounded once to float32 (the table reading the kernels embed)."""
    off = 0.9677083
    pos = [ppf(off + k * (0.5 - off) / 8.0) for k in range(8)]
    neg = [-ppf(off + k * (0.5 - off) / 7.0) for k in range(7)]
    vals = sorted(neg + [0.0] + pos)
    return np.array([v / max(vals) for v in vals], dtype=np.float64).astype(F32)


def test_levels_equal_two_library_builds_bit_for_bit():
    # Python's statistics.NormalDist and scipy's ndtri (Cephes) are written
    # independently of the oracle's AS241; with the exact construction rounded
    # once, all three give the same 16 float32 bit patterns.  L[1] sits 0.497 ulp
    # from a rounding boundary, so a slip in the oracle's quantile, in the
    # offsets' spacing or in the normalisation changes at least one pattern.
    ours = O.nf4_levels().view(np.uint32)
    nd = _levels_from_library_ppf(statistics.NormalDist().inv_cdf).view(np.uint32)
    cephes = _levels_from_library_ppf(lambda p: float(scipy.special.ndtri(p))).view(np.uint32)
    assert np.array_equal(nd, cephes)
    assert np.array_equal(ours, nd), [hex(int(v)) for v in ours]


# ---------------------------------------------------------------------------
# The page's worked example
# ---------------------------------------------------------------------------
def _snippet_weights():
    torch.manual_seed(0)
    return (torch.randn(4096, 64) * 0.02).numpy()


def _mse(w, lv):
    s = O.block_absmax(w)
    c = O.assign_codes(w, s, lv)
    rest = (lv[c].reshape(-1, 64) * s[:, None]).astype(F32)
    return float(np.mean((rest.astype(np.float64) - w.reshape(-1, 64).astype(np.float64)) ** 2)), c


def test_page_example_printed_mse(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "ul_snippet_mse.json")))
    w = _snippet_weights()
    assert w.shape == (g["blocks"], g["block"])
    nf4, _ = _mse(w, O.nf4_levels())
    uni, _ = _mse(w, O.uniform4_levels())
    assert f"{nf4:.3e}" == g["nf4_mse_printed"]
    assert f"{uni:.3e}" == g["uniform4_mse_printed"]
    assert abs((1 - nf4 / uni) - g["relative_reduction_stated"]) < 0.01


def test_page_example_codes_match_torch_argmin():
    # Same data through torch's own float32 argmin with the snippet's level table:
    # every one of the 262144 codes agrees (argmin semantics, ties, float32 math).
    w = _snippet_weights()
    _, ours = _mse(w, O.nf4_levels())
    wt = torch.from_numpy(w)
    am = wt.abs().amax(dim=1, keepdim=True)
    lv = torch.from_numpy(_torch_fp32_levels())
    theirs = ((wt / am)[..., None] - lv).abs().argmin(dim=-1).reshape(-1).numpy()
    assert np.array_equal(ours.astype(np.int64), theirs)


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_nf4_beats_uniform_by_about_16_percent(seed):
    g = torch.Generator().manual_seed(seed)
    w = (torch.randn(8192, 64, generator=g) * 0.02).numpy()
    nf4, _ = _mse(w, O.nf4_levels())
    uni, _ = _mse(w, O.uniform4_levels())
    assert 0.14 < 1 - nf4 / uni < 0.18


# ---------------------------------------------------------------------------
# Code assignment: exact-rational brute force of the float32 definition
# ---------------------------------------------------------------------------
def _fl32(q: Fraction) -> Fraction:
    """Round a rational to the nearest float32 (ties to even), normal/subnormal."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def _brute_codes(block, levels):
    ws = [Fraction(float(v)) for v in block]
    s = max(abs(v) for v in ws)
    lv = [Fraction(float(v)) for v in levels]
    out = []
    for w in ws:
        if s == 0:
            out.append(7)
            continue
        x = _fl32(w / s)
        d = [abs(_fl32(x - l)) for l in lv]
        out.append(min(range(16), key=lambda j: (d[j], j)))
    return out


def test_codes_exact_rational_bruteforce():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((24, 64)) * 0.02).astype(F32)
    w[3] = 0.0                                          # all-zero block
    w[5, :] = np.float32(1e-30) * rng.standard_normal(64).astype(F32)  # tiny scale
    lv = O.nf4_levels()
    got = O.assign_codes(w, O.block_absmax(w), lv).reshape(24, 64)
    for b in range(24):
        assert list(got[b]) == _brute_codes(w[b], lv), b


def _tie_points(levels):
    """float32 x in (L_j, L_j+1) with fl32(x - L_j) == fl32(L_j+1 - x)."""
    pts = []
    for j in range(15):
        lo, hi = Fraction(float(levels[j])), Fraction(float(levels[j + 1]))
        mid = np.float32(float((lo + hi) / 2))
        cand = mid
        for _ in range(8):
            cand = np.nextafter(cand, np.float32(-2))
        for _ in range(17):
            x = Fraction(float(cand))
            if _fl32(x - lo) == _fl32(hi - x):
                pts.append((j, np.float32(cand)))
            cand = np.nextafter(cand, np.float32(2))
    return pts


def test_ties_go_to_lower_level():
    lv = O.nf4_levels()
    ties = _tie_points(lv)
    assert len(ties) >= 3
    for j, x in ties:
        blk = np.zeros(64, F32)
        blk[0] = 1.0                                    # S = 1, so w / S = w exactly
        blk[1] = x
        c = O.assign_codes(blk, O.block_absmax(blk), lv)
        assert c[1] == j, (j, x)


def test_exact_levels_map_to_themselves():
    lv = O.nf4_levels()
    for s in (F32(1.0), F32(0.037), F32(3.5e-4)):
        blk = np.zeros(64, F32)
        blk[:16] = (lv * s).astype(F32)
        blk[16:32] = (lv * s).astype(F32)[::-1]
        c = O.assign_codes(blk, O.block_absmax(blk), lv)
        if s == 1.0:
            assert list(c[:16]) == list(range(16))
        assert c[0] == 0 and c[15] == 15 and c[7] == 7


def test_zero_block_and_zero_group():
    w = np.zeros((2, 64 * 300), F32)                    # 600 blocks -> groups of 256, 256, 88
    w[1, 5] = 0.5
    q = O.quantize(w, 2, 64 * 300)
    codes = O.unpack_codes(q["codes"])
    assert np.all(codes[:300 * 64] == 7)
    assert np.all(q["absmax"][:300] == 0)
    assert q["c2"][0] == 0 and np.all(q["scale_codes"][:256] == 0)
    wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], 2, 64 * 300)
    assert np.all(wd[0] == 0) and not np.any(np.signbit(wd[0]))
    assert wd[1, 5] == 0.5


def test_pack_layout():
    codes = np.array([1, 2, 3, 4, 15, 0], np.uint8)
    p = O.pack_codes(codes)
    assert list(p) == [0x21, 0x43, 0x0F]
    assert np.array_equal(O.unpack_codes(p), codes)


# ---------------------------------------------------------------------------
# OCP FP8 E4M3
# ---------------------------------------------------------------------------
def test_e4m3_spec_points():
    # max normal 1.75*2^8, min normal 2^-6, min subnormal 2^-9, one, ties to even
    assert O.e4m3_encode([448.0])[0] == 0x7E
    assert O.e4m3_encode([2.0 ** -6])[0] == 0x08
    assert O.e4m3_encode([2.0 ** -9])[0] == 0x01
    assert O.e4m3_encode([1.0])[0] == 0x38
    assert O.e4m3_encode([0.0])[0] == 0x00
    assert O.e4m3_encode([1.0625])[0] == 0x38     # halfway 1 .. 1.125 -> even (1.0)
    assert O.e4m3_encode([1.1875])[0] == 0x3A     # halfway 1.125 .. 1.25 -> even (1.25)
    assert O.e4m3_encode([2.0 ** -10])[0] == 0x00  # halfway 0 .. 2^-9 -> even (0)
    assert O.e4m3_encode([1000.0])[0] == 0x7E     # saturates
    assert O.e4m3_decode(0x7E) == 448.0 and np.isnan(O.e4m3_decode(0x7F))
    assert O.e4m3_decode(0x01) == 2.0 ** -9 and O.e4m3_decode(0xB8) == -1.0


def test_e4m3_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    got = O.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, F32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_vs_torch():
    pos = O.e4m3_decode(np.arange(0x7F)).astype(np.float64)
    mids = ((pos[1:] + pos[:-1]) / 2).astype(F32)
    around = [mids]
    for k in range(1, 4):
        around += [np.nextafter(mids, np.float32(1e9)), np.nextafter(mids, np.float32(-1))]
        mids = around[-2]
    probe = np.concatenate(around + [pos.astype(F32)])
    rng = np.random.default_rng(3)
    probe = np.concatenate([probe, np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 400000)).astype(F32),
                            rng.uniform(0, 448.0, 100000).astype(F32)])
    probe = probe[(probe >= 0) & (probe <= 448.0)]
    assert np.array_equal(O.e4m3_encode(probe), _torch_e4m3(probe))


# ---------------------------------------------------------------------------
# Double quantisation and storage size
# ---------------------------------------------------------------------------
def test_double_quant_scale_error_bound():
    rng = np.random.default_rng(11)
    w = (rng.standard_normal(64 * 256 * 3 + 64 * 17) * 0.02).astype(F32)
    q = O.quantize(w, 1, w.size)
    s, sp = q["absmax"], O.dequantize_scales(q["scale_codes"], q["c2"])
    g = np.arange(s.size) // 256
    normal_range = s / q["c2"][g] >= 2.0 ** -6
    rel = np.abs(sp - s) / s
    assert np.all(rel[normal_range] <= 2.0 ** -4 * (1 + 1e-6))
    # the group maximum is encoded at the top of the E4M3 range
    for gi in range(q["c2"].size):
        blk = slice(gi * 256, (gi + 1) * 256)
        assert q["scale_codes"][blk].max() == 0x7E


_E4M3_EXACT = [Fraction(float(v)) for v in O.e4m3_decode(np.arange(0x7F))]  # 0x00 .. 0x7E


def _e4m3_rne_exact(x: Fraction) -> int:
    """E4M3 code of a non-negative rational: nearest value, ties to the code with
    an even last mantissa bit, saturating at 448 (exact arithmetic)."""
    if x >= _E4M3_EXACT[-1]:
        return 0x7E
    hi = next(i for i, v in enumerate(_E4M3_EXACT) if v >= x)
    if _E4M3_EXACT[hi] == x or hi == 0:
        return hi
    lo = hi - 1
    d_lo, d_hi = x - _E4M3_EXACT[lo], _E4M3_EXACT[hi] - x
    if d_lo != d_hi:
        return lo if d_lo < d_hi else hi
    return lo if lo % 2 == 0 else hi


def _near_tie_scales(c2: np.float32, rng) -> np.ndarray:
    """float32 scales S whose quotient S / c2 lies within a few float32 ulps of
    E4M3 rounding midpoints, so that rounding the quotient to float32 first
    (or not) decides the E4M3 code."""
    out = []
    mids = [(a + b) / 2 for a, b in zip(_E4M3_EXACT[:-1], _E4M3_EXACT[1:])]
    for mid in rng.choice(len(mids), 24, replace=False):
        s0 = np.float32(float(mids[mid] * Fraction(float(c2))))
        for k in range(-3, 4):
            s = s0
            for _ in range(abs(k)):
                s = np.nextafter(s, np.float32(np.inf if k > 0 else 0))
            out.append(s)
    return np.array(out, F32)


def test_double_quantize_exact_rational():
    # c2 = fl32(max S / 448) and q = E4M3_rne(fl32(S / c2)), re-derived in exact
    # rational arithmetic on three groups, the last one ragged (100 blocks), with
    # scales placed where the quotient lands on or next to an E4M3 midpoint once
    # rounded to float32: rounding S / c2 in float64, or keeping c2 in float64,
    # changes codes here.
    rng = np.random.default_rng(29)
    groups = []
    for size in (256, 256, 100):
        m = np.float32(rng.uniform(0.01, 0.08))
        c2 = F32(float(_fl32(Fraction(float(m)) / 448)))
        s = _near_tie_scales(c2, rng)
        s = s[(s > 0) & (s < m)][: size - 1]
        fill = (rng.uniform(0.0, 1.0, size - 1 - s.size) * m).astype(F32)
        g = np.concatenate([[m], s, fill]).astype(F32)
        rng.shuffle(g)
        groups.append(g)
    scales = np.concatenate(groups)
    q, c2 = O.double_quantize(scales)
    assert c2.size == 3 and q.size == 612
    mids = {a / 2 + b / 2 for a, b in zip(_E4M3_EXACT[:-1], _E4M3_EXACT[1:])}
    ties_hit = 0
    for gi, g in enumerate(groups):
        m = max(Fraction(float(v)) for v in g)
        c2_exact = _fl32(m / 448)
        assert Fraction(float(c2[gi])) == c2_exact
        for bi, sv in enumerate(g):
            x = _fl32(Fraction(float(sv)) / c2_exact)
            want = _e4m3_rne_exact(x)
            ties_hit += x in mids
            assert q[gi * 256 + bi] == want, (gi, bi, float(sv))
    assert ties_hit >= 5  # the construction really reaches exact float32 midpoints


# ---------------------------------------------------------------------------
# The other readings of the 8-bit scale format: OCP FP8 E5M2 and a linear byte
# ---------------------------------------------------------------------------
def test_e5m2_spec_points():
    # max normal 1.75*2^15, min normal 2^-14, min subnormal 2^-16, one, ties to even
    assert O.e5m2_encode([57344.0])[0] == 0x7B
    assert O.e5m2_encode([2.0 ** -14])[0] == 0x04
    assert O.e5m2_encode([2.0 ** -16])[0] == 0x01
    assert O.e5m2_encode([1.0])[0] == 0x3C
    assert O.e5m2_encode([0.0])[0] == 0x00
    assert O.e5m2_encode([1.125])[0] == 0x3C      # halfway 1 .. 1.25 -> even (1.0)
    assert O.e5m2_encode([1.375])[0] == 0x3E      # halfway 1.25 .. 1.5 -> even (1.5)
    assert O.e5m2_encode([2.0 ** -17])[0] == 0x00  # halfway 0 .. 2^-16 -> even (0)
    assert O.e5m2_encode([1e6])[0] == 0x7B        # saturates
    assert O.e5m2_decode(0x7B) == 57344.0 and O.e5m2_decode(0x7C) == np.inf and np.isnan(O.e5m2_decode(0x7D))
    assert O.e5m2_decode(0x01) == 2.0 ** -16 and O.e5m2_decode(0xBC) == -1.0


def test_e5m2_decode_all_codes_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e5m2).float().numpy().astype(np.float64)
    got = O.e5m2_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_e5m2_encode_vs_torch():
    pos = O.e5m2_decode(np.arange(0x7C)).astype(np.float64)
    mids = ((pos[1:] + pos[:-1]) / 2).astype(F32)
    around = [mids]
    for k in range(1, 4):
        around += [np.nextafter(mids, np.float32(1e9)), np.nextafter(mids, np.float32(-1))]
        mids = around[-2]
    probe = np.concatenate(around + [pos.astype(F32)])
    rng = np.random.default_rng(7)
    probe = np.concatenate([probe, np.exp(rng.uniform(np.log(1e-6), np.log(57344.0), 400000)).astype(F32)])
    probe = probe[(probe >= 0) & (probe <= 57344.0)]   # torch's cast does not saturate; in range it is RNE
    ref = torch.from_numpy(probe).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(O.e5m2_encode(probe), ref)


def test_u8_encode_rounding():
    k = np.arange(256, dtype=np.float64)
    assert np.array_equal(O.u8_encode(k), k.astype(np.uint8))
    half = k[:-1] + 0.5                                   # ties go to the even integer
    assert np.array_equal(O.u8_encode(half), (k[:-1] + (k[:-1] % 2 == 1)).astype(np.uint8))
    up = np.nextafter(half.astype(F32), np.float32(1e9))
    dn = np.nextafter(half.astype(F32), np.float32(-1))
    assert np.array_equal(O.u8_encode(up), (k[:-1] + 1).astype(np.uint8))
    assert np.array_equal(O.u8_encode(dn), k[:-1].astype(np.uint8))
    assert O.u8_encode([255.4999, 255.5, 300.0])[2] == 255 and O.u8_encode([255.5])[0] == 255


def _rne_exact(x: Fraction, table) -> int:
    """Index of the nearest table value (exact rationals, increasing) to x >= 0,
    ties to the even index, saturating at the last entry."""
    if x >= table[-1]:
        return len(table) - 1
    hi = next(i for i, v in enumerate(table) if v >= x)
    if table[hi] == x or hi == 0:
        return hi
    lo = hi - 1
    d_lo, d_hi = x - table[lo], table[hi] - x
    if d_lo != d_hi:
        return lo if d_lo < d_hi else hi
    return lo if lo % 2 == 0 else hi


@pytest.mark.parametrize("fmt", ["e5m2", "u8"])
def test_double_quantize_exact_rational_other_formats(fmt):
    # c2 = fl32(max S / F) and q = enc(fl32(S / c2)), re-derived in exact rational
    # arithmetic, with scales placed where the quotient lands on or next to a
    # rounding midpoint of the format once rounded to float32.
    top = {"e5m2": 0x7B, "u8": 255}[fmt]
    fmax = {"e5m2": 57344, "u8": 255}[fmt]
    table = [Fraction(float(v)) for v in O.scale_decode(np.arange(top + 1), fmt)]
    mids = [(a + b) / 2 for a, b in zip(table[:-1], table[1:])]
    rng = np.random.default_rng(31)
    groups = []
    for size in (256, 256, 100):
        m = np.float32(rng.uniform(0.01, 0.08))
        c2 = F32(float(_fl32(Fraction(float(m)) / fmax)))
        near = []
        for mid in rng.choice(len(mids), 24, replace=False):
            s0 = np.float32(float(mids[mid] * Fraction(float(c2))))
            for kk in range(-3, 4):
                sv = s0
                for _ in range(abs(kk)):
                    sv = np.nextafter(sv, np.float32(np.inf if kk > 0 else 0))
                near.append(sv)
        near = np.array(near, F32)
        near = near[(near > 0) & (near < m)][: size - 1]
        fill = (rng.uniform(0.0, 1.0, size - 1 - near.size) * m).astype(F32)
        g = np.concatenate([[m], near, fill]).astype(F32)
        rng.shuffle(g)
        groups.append(g)
    scales = np.concatenate(groups)
    q, c2 = O.double_quantize(scales, fmt)
    assert c2.size == 3 and q.size == 612
    midset = set(mids)
    ties_hit = 0
    for gi, g in enumerate(groups):
        m = max(Fraction(float(v)) for v in g)
        c2_exact = _fl32(m / fmax)
        assert Fraction(float(c2[gi])) == c2_exact
        assert q[gi * 256: gi * 256 + g.size].max() == top      # the group maximum maps to the top code
        for bi, sv in enumerate(g):
            x = _fl32(Fraction(float(sv)) / c2_exact)
            ties_hit += x in midset
            assert q[gi * 256 + bi] == _rne_exact(x, table), (fmt, gi, bi, float(sv))
    assert ties_hit >= 5


@pytest.mark.parametrize("fmt,bound", [("e5m2", 2.0 ** -3), ("u8", None)])
def test_other_formats_scale_error_bound(fmt, bound):
    rng = np.random.default_rng(12)
    w = (rng.standard_normal(64 * 256 * 3 + 64 * 17) * 0.02).astype(F32)
    q = O.quantize(w, 1, w.size, scale_format=fmt)
    assert q["scale_format"] == fmt
    s, sp = q["absmax"], O.dequantize_scales(q["scale_codes"], q["c2"], fmt)
    g = np.arange(s.size) // 256
    if bound is not None:   # half an ulp of a 2-bit mantissa, in the normal range
        normal_range = s / q["c2"][g] >= 2.0 ** -14
        assert np.all((np.abs(sp - s) / s)[normal_range] <= bound * (1 + 1e-6))
    else:                   # half a step of c2, plus float32 rounding of the product
        assert np.all(np.abs(sp.astype(np.float64) - s) <= q["c2"][g].astype(np.float64) * (0.5 + 1e-5))
    # the dequantised weight uses the format's scales
    wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], 1, w.size, scale_format=fmt)
    lv = O.nf4_levels()
    c = O.unpack_codes(q["codes"])
    assert np.array_equal(wd.reshape(-1), O.bf16_round((lv[c].reshape(-1, 64) * sp[:, None]).astype(F32).reshape(-1)))


def test_storage_overhead_closed_form(golden_dir):
    figs = {f["what"]: f["value"] for f in json.load(open(os.path.join(golden_dir, "memory_figures.json")))["figures"]}
    rows, cols = 4096, 4096
    cb, sb, c2b = O.storage_bytes(rows, cols)
    bits = 8.0 * (cb + sb + c2b) / (rows * cols)
    assert bits == 4 + 8 / 64 + 32 / (64 * 256)                    # 4.126953125 exactly
    overhead = bits - 4
    no_dq = 32 / 64
    assert no_dq == figs["first-level scale overhead without double quantisation, bits per parameter"]
    assert round(overhead, 3) == figs["scale overhead with double quantisation, bits per parameter (about)"]
    saving = no_dq - overhead
    assert round(saving, 2) == figs["saving from double quantisation, bits per parameter (about)"]
    assert round(saving, 1) == figs["saving from nested quantisation, bits per parameter"]
    p65 = 65e9
    assert round(p65 * saving / 8 / 1e9) == figs["saving from double quantisation at 65B parameters, GB (about)"]
    assert round(p65 * 2 / 1e9) == figs["65B weights at 16 bit, GB (about)"]
    gb = p65 * bits / 8 / 1e9                                        # 33.5 GB
    assert abs(gb - figs["65B 4-bit weights plus double-quantised scales, GB (about)"]) <= 0.5
    # the two pages round the same quantity differently (34 vs 33); 33.5 lies between
    assert abs(gb - figs["65B base model in NF4, GB (about)"]) <= 1.0


def test_requantise_is_idempotent():
    rng = np.random.default_rng(5)
    rows, cols = 96, 640
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(F32)
    q = O.quantize(w, rows, cols)
    wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], rows, cols)
    q2 = O.quantize(wd, rows, cols)
    assert np.array_equal(q["codes"], q2["codes"])


def test_dequantize_is_level_times_scale_rounded_once():
    rng = np.random.default_rng(9)
    rows, cols = 8, 256
    w = (rng.standard_normal((rows, cols)) * 0.02).astype(F32)
    q = O.quantize(w, rows, cols)
    wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], rows, cols).reshape(-1)
    codes = O.unpack_codes(q["codes"])
    lv = O.nf4_levels()
    for i in range(0, rows * cols, 37):                 # exact rational re-derivation
        b = i // 64
        sp = _fl32(Fraction(float(O.e4m3_decode(q["scale_codes"][b]))) * Fraction(float(q["c2"][b // 256])))
        prod = _fl32(Fraction(float(lv[codes[i]])) * sp)
        # bf16 RNE of a float32: keep 8 significant bits
        v = float(prod)
        ref = float(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).float())
        assert wd[i] == ref


# ---------------------------------------------------------------------------
# Linear layer with LoRA
# ---------------------------------------------------------------------------
def _tiny_linear(seed=0, m=4, n=8, k=16, r=2):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, k))
    a = rng.standard_normal((r, k))
    b = rng.standard_normal((n, r))
    x = rng.standard_normal((m, k))
    dy = rng.standard_normal((m, n))
    return w, a, b, x, dy


def test_linear_fwd_bruteforce_loops():
    w, a, b, x, _ = _tiny_linear()
    m, k = x.shape
    n, r = b.shape
    alpha = 3.0
    s = alpha / r
    y, t = O.linear_fwd(w, a, b, x, alpha, r)
    for i in range(m):
        for jr in range(r):
            assert abs(t[i, jr] - sum(x[i, kk] * a[jr, kk] for kk in range(k))) < 1e-12
        for j in range(n):
            base = sum(x[i, kk] * w[j, kk] for kk in range(k))
            lora = sum(sum(x[i, kk] * a[jr, kk] for kk in range(k)) * b[j, jr] for jr in range(r))
            assert abs(y[i, j] - (base + s * lora)) < 1e-11


def test_linear_bwd_bruteforce_loops():
    w, a, b, x, dy = _tiny_linear(1)
    m, k = x.shape
    n, r = b.shape
    alpha = 4.0
    s = alpha / r
    dx, da, db = O.linear_bwd(w, a, b, x, dy, alpha, r)
    u = [[sum(dy[i, j] * b[j, jr] for j in range(n)) for jr in range(r)] for i in range(m)]
    t = [[sum(x[i, kk] * a[jr, kk] for kk in range(k)) for jr in range(r)] for i in range(m)]
    for i in range(m):
        for kk in range(k):
            ref = sum(dy[i, j] * w[j, kk] for j in range(n)) + s * sum(u[i][jr] * a[jr, kk] for jr in range(r))
            assert abs(dx[i, kk] - ref) < 1e-11
    for jr in range(r):
        for kk in range(k):
            assert abs(da[jr, kk] - s * sum(u[i][jr] * x[i, kk] for i in range(m))) < 1e-11
    for j in range(n):
        for jr in range(r):
            assert abs(db[j, jr] - s * sum(dy[i, j] * t[i][jr] for i in range(m))) < 1e-11


def test_gradients_by_central_differences():
    w, a, b, x, dy = _tiny_linear(2, m=3, n=5, k=7, r=2)
    alpha, r = 2.0, 2

    def loss(xx, aa, bb):
        y, _ = O.linear_fwd(w, aa, bb, xx, alpha, r)
        return float(np.sum(dy * y))

    dx, da, db = O.linear_bwd(w, a, b, x, dy, alpha, r)
    h = 1e-3
    for arr, grad, which in ((x, dx, 0), (a, da, 1), (b, db, 2)):
        for idx in np.ndindex(arr.shape):
            p, mi = [x.copy(), a.copy(), b.copy()], [x.copy(), a.copy(), b.copy()]
            p[which][idx] += h
            mi[which][idx] -= h
            fd = (loss(*p) - loss(*mi)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-8 * max(1.0, abs(fd))


def test_b_zero_reduces_to_base_layer():
    w, a, b, x, dy = _tiny_linear(3)
    b0 = np.zeros_like(b)
    y, _ = O.linear_fwd(w, a, b0, x, 16.0, 2)
    assert np.array_equal(y, x @ w.T)
    dx, da, db = O.linear_bwd(w, a, b0, x, dy, 16.0, 2)
    assert np.all(da == 0)
    assert np.array_equal(dx, dy @ w)


def test_w_zero_isolates_lora_path():
    w, a, b, x, _ = _tiny_linear(4)
    y, t = O.linear_fwd(np.zeros_like(w), a, b, x, 16.0, 2)
    assert np.allclose(y, 8.0 * (x @ a.T) @ b.T, rtol=0, atol=1e-12)


def test_merged_form_agrees():
    w, a, b, x, _ = _tiny_linear(5, m=6, n=9, k=20, r=3)
    y, _ = O.linear_fwd(w, a, b, x, 6.0, 3)
    wm = O.merged_weight(w, a, b, 6.0, 3)
    assert np.allclose(y, x @ wm.T, rtol=1e-13, atol=1e-13)


def test_lora_scale_float32():
    assert O.lora_scale(16.0, 8) == 2.0
    assert O.lora_scale(16.0, 64) == 0.25
    assert O.lora_scale(1.0, 3) == float(np.float32(1.0) / np.float32(3.0))


# ---------------------------------------------------------------------------
# Merged export and the adapter optimiser step
# ---------------------------------------------------------------------------
def _quantised(n, k, seed, scale=0.02):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((n, k)) * scale).astype(np.float32)
    q = O.quantize(w, n, k)
    return q, O.dequantize(q["codes"], q["scale_codes"], q["c2"], n, k)


def test_merge_export_with_b_zero_is_the_dequantised_weight():
    q, wd = _quantised(24, 128, 11)
    a = np.random.default_rng(1).standard_normal((8, 128)).astype(np.float32)
    got = O.merge_export(q["codes"], q["scale_codes"], q["c2"], 24, 128, a, np.zeros((24, 8), np.float32), 16.0, 8)
    assert np.array_equal(got.view(np.uint32), wd.astype(np.float32).view(np.uint32))


def test_merge_export_with_w_zero_is_one_bf16_rounding_of_the_update():
    # integer-valued B and A small enough that s B A is exact in float32, so the
    # float32 -> bf16 cast of torch (round to nearest even) is the reference
    n, k, r = 16, 64, 8
    rng = np.random.default_rng(2)
    a = rng.integers(-300, 300, (r, k)).astype(np.float32)
    b = rng.integers(-300, 300, (n, r)).astype(np.float32)
    q = O.quantize(np.zeros((n, k), np.float32), n, k)
    got = O.merge_export(q["codes"], q["scale_codes"], q["c2"], n, k, a, b, 16.0, r)
    exact = (2.0 * (b.astype(np.float64) @ a.astype(np.float64))).astype(np.float32)
    assert np.array_equal(exact.astype(np.float64), 2.0 * (b.astype(np.float64) @ a.astype(np.float64)))
    want = torch.from_numpy(exact).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got, want)
    assert np.any(got != exact)  # the rounding is exercised


def test_merged_export_reproduces_the_layer_forward():
    q, wd = _quantised(32, 192, 3)
    rng = np.random.default_rng(4)
    a = (rng.standard_normal((8, 192)) / math.sqrt(192)).astype(np.float32)
    b = (rng.standard_normal((32, 8)) * 0.01).astype(np.float32)
    x = rng.standard_normal((5, 192)).astype(np.float32)
    wm = O.merge_export(q["codes"], q["scale_codes"], q["c2"], 32, 192, a, b, 16.0, 8)
    y, _ = O.linear_fwd(wd, a, b, x, 16.0, 8)
    ym = x.astype(np.float64) @ wm.astype(np.float64).T
    # the only difference is the merged weight's own bf16 rounding (2^-9 relative)
    assert np.max(np.abs(ym - y)) <= 2.0 ** -8 * np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=1)).max() * \
        np.abs(wm).max()


def _adamw_torch(p0, grads, lr, b1, b2, eps, wd):
    p = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([p], lr=lr, betas=(b1, b2), eps=eps, weight_decay=wd)
    for g in grads:
        p.grad = torch.from_numpy(g.copy())
        opt.step()
    st = opt.state[p]
    return p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy()


def test_adamw_step_matches_torch_adamw_over_several_steps():
    rng = np.random.default_rng(5)
    p0 = rng.standard_normal(257)
    grads = [rng.standard_normal(257) * (0.1 + i) for i in range(6)]
    hp = dict(lr=3e-3, beta1=0.9, beta2=0.97, eps=1e-7, weight_decay=0.05)
    p, m, v = p0, np.zeros_like(p0), np.zeros_like(p0)
    for t, g in enumerate(grads, start=1):
        p, m, v = O.adamw_step(p, g, m, v, t, **hp)
    tp, tm, tv = _adamw_torch(p0, grads, hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    assert np.allclose(p, tp, rtol=1e-12, atol=1e-14)
    assert np.allclose(m, tm, rtol=1e-12, atol=1e-14)
    assert np.allclose(v, tv, rtol=1e-12, atol=1e-14)


def test_adamw_step_closed_forms():
    rng = np.random.default_rng(6)
    p0 = rng.standard_normal(64)
    # zero gradient and zero state: only the decoupled decay acts
    p, m, v = O.adamw_step(p0, np.zeros(64), np.zeros(64), np.zeros(64), 1, 1e-2, 0.9, 0.999, 1e-8, 0.1)
    assert np.array_equal(p, p0 * (1.0 - 1e-3)) and not m.any() and not v.any()
    # first step without decay: the bias corrections cancel, the step is lr g / (|g| + eps)
    g = rng.standard_normal(64)
    p, _, _ = O.adamw_step(p0, g, np.zeros(64), np.zeros(64), 1, 1e-2, 0.9, 0.999, 1e-8, 0.0)
    assert np.allclose(p, p0 - 1e-2 * g / (np.abs(g) + 1e-8), rtol=1e-14, atol=1e-16)


def test_adamw_pin_catches_a_planted_sign_error():
    rng = np.random.default_rng(7)
    p0, g = rng.standard_normal(32), rng.standard_normal(32)
    good, _, _ = O.adamw_step(p0, g, np.zeros(32), np.zeros(32), 1, 1e-2, 0.9, 0.999, 1e-8, 0.0)
    bad = p0 + 1e-2 * g / (np.abs(g) + 1e-8)  # the update applied with the wrong sign
    tp, _, _ = _adamw_torch(p0, [g], 1e-2, 0.9, 0.999, 1e-8, 0.0)
    assert np.allclose(good, tp) and not np.allclose(bad, tp)


def test_multi_adapter_forward_reduces_and_separates():
    w, a, b, x, _ = _tiny_linear(8, m=5, n=9, k=20, r=3)
    rng = np.random.default_rng(9)
    a2, b2 = rng.standard_normal(a.shape), rng.standard_normal(b.shape)
    ads = [(a, b, 6.0, 3), (a2, b2, 2.0, 3)]
    # one adapter for every token: the single-adapter forward (row-by-row and
    # batched products differ only in float64 summation order)
    y1, _ = O.linear_fwd(w, a, b, x, 6.0, 3)
    assert np.allclose(O.linear_fwd_multi(w, ads, [0] * 5, x), y1, rtol=1e-13, atol=1e-13)
    # a token's output depends only on its own adapter
    idx = [1, 0, 1, 1, 0]
    ym = O.linear_fwd_multi(w, ads, idx, x)
    y2, _ = O.linear_fwd(w, a2, b2, x, 2.0, 3)
    for t, i in enumerate(idx):
        assert np.allclose(ym[t], (y1 if i == 0 else y2)[t], rtol=1e-13, atol=1e-13)
    # and two different adapters give different outputs
    assert not np.allclose(ym[0], y1[0])


def _dropout_case(seed, m=6, n=9, k=24, r=3, p=0.25):
    rng = np.random.default_rng(seed)
    w, a, b, x, dy = _tiny_linear(seed, m=m, n=n, k=k, r=r)
    keep = rng.random((m, k)) >= p
    return w, a, b, x, dy, keep, p


def test_keep_mask_packing_layout():
    rng = np.random.default_rng(1)
    keep = rng.random((3, 40)) < 0.5
    packed = np.zeros((3, 5), np.uint8)
    for i in range(3):
        for j in range(40):
            if keep[i, j]:
                packed[i, j // 8] |= np.uint8(1 << (j % 8))
    assert np.array_equal(O.unpack_keep(packed, 3, 40), keep)


def test_dropout_with_nothing_dropped_is_the_plain_layer():
    w, a, b, x, dy, _, _ = _dropout_case(2)
    keep = np.ones(x.shape, bool)
    y, t = O.linear_fwd_dropout(w, a, b, x, keep, 0.0, 6.0, 3)
    y0, t0 = O.linear_fwd(w, a, b, x, 6.0, 3)
    assert np.allclose(y, y0, rtol=1e-14, atol=1e-14) and np.allclose(t, t0, rtol=1e-14, atol=1e-14)
    for g1, g0 in zip(O.linear_bwd_dropout(w, a, b, x, dy, keep, 0.0, 6.0, 3), O.linear_bwd(w, a, b, x, dy, 6.0, 3)):
        assert np.allclose(g1, g0, rtol=1e-13, atol=1e-13)


def test_dropout_with_everything_dropped_removes_the_adapter():
    w, a, b, x, dy, _, p = _dropout_case(3)
    keep = np.zeros(x.shape, bool)
    y, t = O.linear_fwd_dropout(w, a, b, x, keep, p, 6.0, 3)
    assert not t.any() and np.allclose(y, x @ w.T, rtol=1e-14, atol=1e-14)
    dx, da, db = O.linear_bwd_dropout(w, a, b, x, dy, keep, p, 6.0, 3)
    assert not da.any() and not db.any() and np.allclose(dx, dy @ w, rtol=1e-14, atol=1e-14)


def test_dropout_gradients_by_finite_differences():
    w, a, b, x, dy, keep, p = _dropout_case(4)

    def loss(x_, a_, b_):
        y, _ = O.linear_fwd_dropout(w, a_, b_, x_, keep, p, 6.0, 3)
        return float(np.sum(y * dy))

    dx, da, db = O.linear_bwd_dropout(w, a, b, x, dy, keep, p, 6.0, 3)
    h = 1e-6
    for arr, grad, which in ((x, dx, 0), (a, da, 1), (b, db, 2)):
        for idx in [(0, 0), (1, 2), (arr.shape[0] - 1, arr.shape[1] - 1), (2, arr.shape[1] // 2)]:
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = [x, a, b]
            args_m = [x, a, b]
            args_p[which], args_m[which] = plus, minus
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-6 * max(1.0, abs(fd))
