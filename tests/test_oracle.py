"""Pins for the CPU oracle, against references other than itself.

Every check here runs on the CPU.  The references are: numpy's and torch's own
float16 / bfloat16 conversions, the E2M1 bit-field definition, exact grid
round-trips, brute-force enumeration on tiny groups, hand-worked fixtures under
tests/golden/, and numpy float64 matrix products for the reference GEMV/GEMM.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from dequant_gemv_rtn_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ conversions
def test_h2d_all_fp16_patterns(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = orc.h2d(bits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # sign of zero
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _check_f2h_chunk(orc, lo, hi):
    u = np.arange(lo, hi, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    got = orc.f2h(f)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan]), (lo, hi)
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


@pytest.mark.skipif(os.environ.get("QNT_EXHAUSTIVE") != "1", reason="set QNT_EXHAUSTIVE=1 (about 5 min)")
def test_f2h_exhaustive_positive_range(orc):
    """All 2^31 non-negative binary32 patterns vs numpy's float32->float16 (RNE)."""
    step = 1 << 26
    for lo in range(0, 1 << 31, step):
        _check_f2h_chunk(orc, lo, lo + step)


def test_f2h_structured_sample(orc):
    """Every sign and exponent, with low mantissa bits set around every possible
    rounding position (normal fp16: bit 13; fp16 subnormals: bits 14..24)."""
    rng = np.random.default_rng(1)
    hi = np.concatenate([np.array([0, 1, 0x3FE, 0x3FF], np.uint32), rng.integers(0, 1024, 60).astype(np.uint32)])
    lows = set()
    for k in range(12, 24):
        for v in (0, 1, (1 << (k - 1)) - 1, 1 << (k - 1), (1 << (k - 1)) + 1, (1 << k) - 1):
            lows.add(v)
    lows = np.array(sorted(lows), np.uint32)
    sign = np.array([0, 1], np.uint32)[:, None, None, None] << 31
    exp = np.arange(256, dtype=np.uint32)[None, :, None, None] << 23
    man = (hi[None, None, :, None] << 13) ^ lows[None, None, None, :]
    u = (sign | exp | (man & 0x7FFFFF)).reshape(-1)
    f = u.view(np.float32)
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    got = orc.f2h(f)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan])


def test_f2h_negative_sample(orc):
    """Negative patterns: sign symmetry plus a dense sample of the fp16 range."""
    _check_f2h_chunk(orc, 0x80000000 + 0x33000000 - (1 << 20), 0x80000000 + 0x33000000 + (1 << 20))
    _check_f2h_chunk(orc, 0x80000000 + 0x38800000, 0x80000000 + 0x38800000 + (1 << 22))
    _check_f2h_chunk(orc, 0x80000000 + 0x477FE000, 0x80000000 + 0x47800000 + (1 << 16))


def test_f2bf_vs_torch(orc):
    rng = np.random.default_rng(3)
    u = np.concatenate([
        rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32),
        np.arange(0x7F7F0000, 0x7F800100, dtype=np.uint32),          # near max / inf
        np.arange(0x00000000, 0x00020000, dtype=np.uint32),          # subnormals
        np.arange(0x3F7F0000, 0x3F810000, dtype=np.uint32),          # around 1.0
    ])
    f = u.view(np.float32)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.f2bf(f)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------------ E2M1 table
def _e2m1_from_bits(code):
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def test_e2m1_table_closed_form(orc):
    for c in range(16):
        assert orc.e2m1(c) == _e2m1_from_bits(c)
        assert math.copysign(1.0, orc.e2m1(c)) == math.copysign(1.0, _e2m1_from_bits(c))


def test_e2m1_table_golden(orc):
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_table.txt")) if l.strip() and not l.startswith("#")]
    assert len(rows) == 16
    for code, val in rows:
        assert orc.e2m1(int(code)) == float(val)


def test_e2m1_table_vs_torch_float4():
    """torch's own float4_e2m1fn_x2 decode, where this torch build provides it."""
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("torch has no float4_e2m1fn_x2")
    from oracle import oracle as orc
    try:
        packed = torch.arange(16, dtype=torch.uint8) | (torch.arange(16, dtype=torch.uint8) << 4)
        vals = packed.view(torch.float4_e2m1fn_x2).to(torch.float32)
    except Exception as e:  # this PyTorch version lacks the conversion
        pytest.skip(f"no float4 conversion: {e}")
    for c in range(16):
        assert float(vals.reshape(-1)[2 * c]) == orc.e2m1(c)


# ------------------------------------------------------------------ golden INT4 example
def test_int4_hand_worked_group(orc):
    rows = [l for l in open(os.path.join(GOLDEN, "int4_group_example.txt")) if l.strip() and not l.startswith("#")]
    w = np.array([float(v) for v in rows[0].split()], np.float32)
    sb, z = rows[1].split()
    codes = [int(v) for v in rows[2].split()]
    c, s1, _, zz, st = orc.quantize_group(orc.INT4, w)
    assert st == 0
    assert s1 == int(sb, 16) and zz == int(z)
    assert list(c) == codes


# ------------------------------------------------------------------ exact grid round-trips
def _rand_fp16_scales(rng, n, lo=-12, hi=2):
    e = rng.integers(lo, hi, size=n)
    m = rng.integers(0, 1024, size=n)
    return (1.0 + m / 1024.0) * np.exp2(e)


@pytest.mark.parametrize("g", [32, 64, 128])
def test_int4_grid_roundtrip(orc, g):
    rng = np.random.default_rng(g)
    N, K = 24, 4 * g
    G = K // g
    s = _rand_fp16_scales(rng, N * G).reshape(N, G)
    z = rng.integers(0, 16, size=(N, G))
    q = rng.integers(0, 16, size=(N, K))
    q[:, ::g] = 0
    q[:, 1::g] = 15
    W = ((q.reshape(N, G, g) - z[..., None]) * s[..., None]).reshape(N, K).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), ((q.reshape(N, G, g) - z[..., None]) * s[..., None]).reshape(N, K))
    r = orc.quantize(orc.INT4, W, g)
    assert r.status == 0
    assert np.array_equal(r.codes, q.astype(np.uint8))
    assert np.array_equal(r.z.reshape(N, G), z.astype(np.uint8))
    assert np.array_equal(orc.h2d(r.s1).reshape(N, G), s)


@pytest.mark.parametrize("fmt", ["fp4", "afpq"])
def test_fp4_grid_roundtrip(orc, fmt):
    rng = np.random.default_rng(7)
    N, g = 16, 128
    K = 2 * g
    mags = np.array([_e2m1_from_bits(c) for c in range(16)])
    codes = rng.integers(0, 16, size=(N, K))
    codes[codes == 8] = 0                     # -0 is never emitted
    codes[:, ::g] = 7                         # +6 present in every group
    codes[:, 1::g] = 15                       # -6 present in every group
    sp = _rand_fp16_scales(rng, N * 2).reshape(N, 2)
    sn = sp if fmt == "fp4" else _rand_fp16_scales(rng, N * 2).reshape(N, 2)
    v = mags[codes].reshape(N, 2, g)
    W = np.where(v > 0, v * sp[..., None], v * sn[..., None]).reshape(N, K)
    r = orc.quantize(orc.FP4 if fmt == "fp4" else orc.AFPQ, W.astype(np.float32), g)
    assert r.status == 0
    assert np.array_equal(r.codes, codes.astype(np.uint8))
    assert np.array_equal(orc.h2d(r.s1).reshape(N, 2), sp)
    if fmt == "afpq":
        assert np.array_equal(orc.h2d(r.s2).reshape(N, 2), sn)


def test_int8_grid_roundtrip(orc):
    rng = np.random.default_rng(11)
    N, K = 8, 256
    s = _rand_fp16_scales(rng, N)
    q = rng.integers(-127, 128, size=(N, K))
    q[:, 0] = 127
    W = (q * s[:, None]).astype(np.float32)
    r = orc.quantize(orc.INT8, W, K)
    assert r.status == 0
    assert np.array_equal(r.codes.view(np.int8), q.astype(np.int8))
    assert np.array_equal(orc.h2d(r.s1), s)


def test_fp16_format_is_rounding(orc):
    W = synth.llama_like(4, 256, seed=5)
    r = orc.quantize(orc.FP16, W, 256)
    assert np.array_equal(r.codes, W.astype(np.float16).view(np.uint16))


# ------------------------------------------------------------------ brute force on tiny groups
def _all_values(fmt, s1, s2, z):
    """Every representable dequantized value of one group, by code (brute force)."""
    vals = {}
    S1 = float(np.uint16(s1).view(np.float16))
    S2 = float(np.uint16(s2).view(np.float16))
    for c in range(16):
        if fmt == 1:
            vals[c] = (c - z) * S1
        elif fmt == 2:
            if c == 8:
                continue
            vals[c] = _e2m1_from_bits(c) * S1
        elif fmt == 3:
            if c == 8:
                continue
            v = _e2m1_from_bits(c)
            vals[c] = v * (S1 if v > 0 else S2)
        elif fmt == 4:
            vals[c] = ([5.0, -5.0, 8.0, -8.0][z] if c == 8 else _e2m1_from_bits(c)) * S1
    return vals


@pytest.mark.parametrize("fmt", [1, 2, 3, 4])
@pytest.mark.parametrize("g", [4, 8])
def test_codes_are_nearest_brute_force(orc, fmt, g):
    """For the stored metadata, each code is the nearest representable value.

    AFPQ restricts each weight to its own sign's half-grid (positive weights to
    s+ values, negative weights to s- values)."""
    rng = np.random.default_rng(100 * fmt + g)
    for trial in range(300):
        w = (rng.standard_t(5, size=g) * 0.02).astype(np.float32)
        codes, s1, s2, z, st = orc.quantize_group(fmt, w)
        assert st == 0
        vals = _all_values(fmt, s1, s2, z)
        for i in range(g):
            x = float(w[i])
            cand = vals
            if fmt == 3:
                cand = {c: v for c, v in vals.items() if (v >= 0) == (x >= 0) or v == 0}
            best = min(abs(x - v) for v in cand.values())
            got = abs(x - vals[int(codes[i])])
            # a division rounding can only flip a choice within one binary32 ulp of a tie
            assert got <= best + 4 * np.spacing(np.float32(abs(x) + best)), (fmt, trial, i, x, codes[i], vals)


def test_fp4_ties_round_to_even(orc):
    """Weights exactly at E2M1 midpoints go to the even-mantissa code."""
    S = 1.0
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    want = [0, 2, 2, 4, 4, 6, 6]              # codes: 0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0
    w = np.array([6.0 * S] + mids, np.float32)
    codes, s1, _, _, st = orc.quantize_group(orc.FP4, w)
    assert s1 == 0x3C00
    assert list(codes[1:]) == want
    codes, _, _, _, _ = orc.quantize_group(orc.FP4, -w)
    assert list(codes[1:]) == [0] + [c | 8 for c in want[1:]]


def test_int4_invariants_and_order_independence(orc):
    rng = np.random.default_rng(5)
    W = synth.llama_like(64, 256, seed=9)
    r = orc.quantize(orc.INT4, W, 128)
    dq = orc.dequant(r)
    S = orc.h2d(r.s1).reshape(64, 2)
    # groups that straddle zero: every weight is within one step of its value
    for n in range(64):
        for j in range(2):
            w = W[n, 128 * j:128 * (j + 1)].astype(np.float64)
            err = np.abs(w - dq[n, 128 * j:128 * (j + 1)])
            assert err.max() <= 1.0 * S[n, j] + 1e-12
    # permuting weights inside a group permutes codes, leaves metadata alone
    for fmt in (orc.INT4, orc.FP4, orc.AFPQ):
        perm = rng.permutation(128)
        Wp = W.copy()
        Wp[:, :128] = W[:, perm]
        a, b = orc.quantize(fmt, W, 128), orc.quantize(fmt, Wp, 128)
        assert np.array_equal(a.s1, b.s1) and np.array_equal(a.s2, b.s2) and np.array_equal(a.z, b.z)
        assert np.array_equal(a.codes[:, perm], b.codes[:, :128])


def test_int4_half_step_bound(orc):
    """|w - dq| <= s/2 whenever rint(w/s)+z lands in [0, 15] without clamping."""
    W = synth.llama_like(32, 512, seed=2)
    r = orc.quantize(orc.INT4, W, 128)
    dq = orc.dequant(r)
    S = np.repeat(orc.h2d(r.s1).reshape(32, 4), 128, axis=1)
    Z = np.repeat(r.z.reshape(32, 4).astype(np.float64), 128, axis=1)
    unclamped = (np.rint(W / S) + Z >= 0) & (np.rint(W / S) + Z <= 15)
    err = np.abs(W.astype(np.float64) - dq)
    assert np.all(err[unclamped] <= 0.5 * S[unclamped] * (1 + 2 ** -20))


# ------------------------------------------------------------------ RaZeR selection
def _razer_brute(w):
    """Brute force: each selector's fp16 scale, nearest codes, plain SSE; argmin."""
    am = np.float32(np.max(np.abs(w)))
    best = None
    for sel, sv in enumerate([5.0, -5.0, 8.0, -8.0]):
        denom = np.float32(max(6.0, abs(sv)))
        s = np.float32(am / denom).astype(np.float16)
        if float(s) == 0.0:
            s = np.float16(1.0)
        S = float(s)
        grid = [(c, (sv if c == 8 else _e2m1_from_bits(c)) * S) for c in range(16)]
        sse = 0.0
        codes = []
        for x in w.astype(np.float64):
            d = [abs(x - v) for _, v in grid]
            c = int(np.argmin(d))
            codes.append(c)
            sse += (x - grid[c][1]) ** 2
        if best is None or sse < best[0]:
            best = (sse, sel, s.view(np.uint16), codes)
    return best


def test_razer_selection_brute_force(orc):
    rng = np.random.default_rng(21)
    checked = 0
    for trial in range(400):
        g = [4, 8, 16][trial % 3]
        w = (rng.standard_t(5, size=g) * 0.02).astype(np.float32)
        codes, s1, _, sel, st = orc.quantize_group(orc.RAZER, w)
        bsse, bsel, bs, _ = _razer_brute(w)
        # recompute the oracle's SSE for its own choice; it must equal the minimum
        S = float(np.uint16(s1).view(np.float16))
        sv = [5.0, -5.0, 8.0, -8.0][sel]
        dq = np.array([(sv if c == 8 else _e2m1_from_bits(int(c))) * S for c in codes])
        osse = float(np.sum((w.astype(np.float64) - dq) ** 2))
        assert osse <= bsse * (1 + 1e-9) + 1e-30, (trial, sel, bsel)
        if abs(osse - bsse) > 1e-6 * bsse:
            continue
        checked += 1
    assert checked > 300


def test_razer_constructed_groups(orc):
    S = 2.0 ** -6
    # on-grid group whose maximum is +8 S: selector +8 (2) reconstructs exactly
    w = np.array([8, 6, -4, 0.5, 1, -1.5, 3, -6], np.float32) * S
    codes, s1, _, sel, _ = orc.quantize_group(orc.RAZER, w)
    assert sel == 2 and s1 == np.float16(S).view(np.uint16)
    assert codes[0] == 8
    # on-grid group (absmax 6 S) containing -5 S: selector -5 (1), exact
    w = np.array([6, -5, -4, 0.5, 1, -1.5, 3, 2], np.float32) * S
    codes, s1, _, sel, _ = orc.quantize_group(orc.RAZER, w)
    assert sel == 1 and codes[1] == 8
    # group on the plain FP4 grid with absmax 6: all +-5 candidates tie -> selector 0
    w = np.array([6, -4, 0.5, 1, -1.5, 3, 2, 0], np.float32) * S
    codes, s1, _, sel, _ = orc.quantize_group(orc.RAZER, w)
    assert sel == 0 and 8 not in list(codes)
    # a weight exactly between 4 S and the special +5 S goes to the regular value
    w = np.array([6, 4.5, 5, 0, 0, 0, 0, 0], np.float32) * S
    codes, s1, _, sel, _ = orc.quantize_group(orc.RAZER, w)
    assert sel == 0 and codes[1] == 6 and codes[2] == 8


def test_afpq_one_sided_and_symmetric(orc):
    w = -np.abs(synth.llama_like(1, 128, seed=4)[0]) - 1e-3
    codes, sp, sn, _, st = orc.quantize_group(orc.AFPQ, w)
    assert sp == 0x3C00                        # no positive weight: s+ defaults to 1
    assert all(c == 0 or c >= 9 for c in codes)
    v = synth.llama_like(1, 64, seed=6)[0]
    w = np.concatenate([v, -v]).astype(np.float32)
    ca, sp, sn, _, _ = orc.quantize_group(orc.AFPQ, w)
    cf, s, _, _, _ = orc.quantize_group(orc.FP4, w)
    assert sp == sn == s and np.array_equal(ca, cf)


# ------------------------------------------------------------------ reference GEMV / GEMM
@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5, 6])
def test_gemm_matches_numpy_float64(orc, fmt):
    N, K = 48, 256
    W = synth.llama_like(N, K, seed=fmt)
    q = orc.quantize(fmt, W, 64 if fmt in orc.FOUR_BIT else K)
    X = synth.activations(3, K, seed=fmt)
    Xh = orc.f2h(X)
    Y, A = orc.gemm(q, Xh, 0)
    D = orc.dequant(q)
    Xd = Xh.view(np.float16).astype(np.float64)
    ref = Xd @ D.T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-300)
    assert np.allclose(A, np.abs(Xd) @ np.abs(D).T, rtol=1e-12)
    # M-batched result equals stacked single-vector results
    for m in range(3):
        y1, _ = orc.gemm(q, Xh[m:m + 1], 0)
        assert np.array_equal(y1[0], Y[m])


def test_gemm_one_hot_and_ones(orc):
    N, K = 40, 256
    W = synth.llama_like(N, K, seed=8)
    q = orc.quantize(orc.INT4, W, 128)
    D = orc.dequant(q)
    for k in [0, 1, 77, 128, 255]:
        x = np.zeros((1, K), np.float32)
        x[0, k] = 1.0
        Y, _ = orc.gemm(q, orc.f2h(x), 0)
        assert np.array_equal(Y[0], D[:, k])
    Y, _ = orc.gemm(q, orc.f2bf(np.ones((1, K), np.float32)), 1)
    assert np.allclose(Y[0], D.sum(axis=1), rtol=1e-13)


def test_int8_group_k_is_per_channel(orc):
    W = synth.llama_like(8, 256, seed=3)
    r = orc.quantize(orc.INT8, W, 256)
    am = np.abs(W).max(axis=1)
    assert np.array_equal(r.s1, (am / np.float32(127)).astype(np.float32).astype(np.float16).view(np.uint16))


# ------------------------------------------------------------------ layout
@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5, 6])
def test_pack_unpack_roundtrip(orc, fmt):
    N, K, g = 5, 384, 64
    W = synth.llama_like(N, K, seed=12)
    q = orc.quantize(fmt, W, g)
    pc, pm = orc.pack(q)
    assert pc.size == orc.codes_bytes(fmt, N, K)
    u = orc.unpack(fmt, N, K, g, pc, pm)
    assert np.array_equal(u.codes, q.codes)
    assert np.array_equal(u.s1, q.s1)
    if fmt == orc.AFPQ:
        assert np.array_equal(u.s2, q.s2)
    if fmt in (orc.INT4, orc.RAZER):
        assert np.array_equal(u.z, q.z)


def test_layout_hand_positions(orc):
    """A few byte/nibble positions worked out by hand from the layout text."""
    N, K, g = 2, 256, 128                      # one row group of 8 rows, 4K = 1024 bytes
    # INT4, weight (n=1, k=187): row group 0, row i=1, block 1, chunk c=1, chunk weight 27:
    # p%2 = 1, r = 11 -> word 2, (p/2)%2 = 1, p/4 = 1 -> p = 7;
    # byte = 512*1 + 64*1 + 16*(1 ^ 0) + 4*2 + 3 = 603, high nibble.
    # FP4, weight (n=1, k=183): block 1, chunk 1, chunk weight 23 -> word 2, p = 7 -> byte 603.
    for fmt, k in [(orc.INT4, 187), (orc.FP4, 183)]:
        codes = np.zeros((N, K), np.uint8)
        codes[1, k] = 0xB
        q = orc.Quant(fmt, N, K, g, codes, np.zeros(4, np.uint16), np.zeros(4, np.uint16), np.zeros(4, np.uint8))
        pc, _ = orc.pack(q)
        assert pc.size == 1024
        assert pc[603] == 0xB0 and pc.sum() == 0xB0
    # INT4 low-nibble half, row 0, chunk 2: k = 76..79 -> word 3, p = 0, 4, 2, 6 -> bytes 44, 46, 45, 47
    for k, byte in [(64 + 12 + 1, 46), (64 + 12 + 2, 45), (64 + 12 + 3, 47), (64 + 12, 44)]:
        codes = np.zeros((N, K), np.uint8)
        codes[0, k] = 0x6
        q = orc.Quant(orc.INT4, N, K, g, codes, np.zeros(4, np.uint16), np.zeros(4, np.uint16), np.zeros(4, np.uint8))
        pc, _ = orc.pack(q)
        assert pc[byte] == 0x06 and pc.sum() == 6, (k, byte)
    # chunk swizzle in the second row group: n = 13 -> group 1, row i = 5, (i/2)%4 = 2;
    # k = 44 -> block 0, chunk 1 -> chunk position 1 ^ 2 = 3;
    # FP4: chunk weight 12 -> word 1, p = 4 -> byte 1024 + 64*5 + 16*3 + 4 + 2 = 1398, low nibble
    # INT4: chunk weight 12 -> p%2 = 0, r = 12 -> word 3, p = 0 -> byte 1024 + 320 + 48 + 12 = 1404, low
    N2 = 14
    for fmt, byte in [(orc.FP4, 1398), (orc.INT4, 1404)]:
        codes = np.zeros((N2, K), np.uint8)
        codes[13, 44] = 0x9
        G2 = N2 * 2
        q = orc.Quant(fmt, N2, K, g, codes, np.zeros(G2, np.uint16), np.zeros(G2, np.uint16), np.zeros(G2, np.uint8))
        pc, _ = orc.pack(q)
        assert pc.size == 16 * 128
        assert pc[byte] == 0x09 and pc.sum() == 9
    # last weight of a K = 4224 row (33 blocks): k = 4223 -> block 32, chunk 3, chunk weight 31;
    # INT4 and FP4 both put it in word 3, p = 7 -> byte 512*32 + 16*3 + 12 + 3 = 16447, high nibble
    K2 = 4224
    G2 = K2 // 128
    for fmt in (orc.INT4, orc.FP4):
        codes = np.zeros((1, K2), np.uint8)
        codes[0, K2 - 1] = 0x5
        q = orc.Quant(fmt, 1, K2, 128, codes, np.zeros(G2, np.uint16), np.zeros(G2, np.uint16), np.zeros(G2, np.uint8))
        pc, _ = orc.pack(q)
        assert pc.size == 8 * K2 // 2
        assert pc[16447] == 0x50 and pc.sum() == 0x50
        codes[:] = 0
        codes[0, 0] = 0x7                       # weight 0 -> byte 0, low nibble (both formats)
        pc, _ = orc.pack(q)
        assert pc[0] == 0x07 and pc.sum() == 7
    # metadata: INT4 zero of group f=3 -> byte round_up(2*4, 256) + 1, high nibble
    q = orc.Quant(orc.INT4, N, K, g, np.zeros((N, K), np.uint8), np.arange(4, dtype=np.uint16),
                  np.zeros(4, np.uint16), np.array([0, 0, 0, 9], np.uint8))
    _, pm = orc.pack(q)
    assert pm[256 + 1] == 0x90 and pm[6] == 3 and pm[7] == 0


def test_nonfinite_weights_reported(orc):
    W = synth.llama_like(4, 128, seed=1)
    W[2, 5] = np.nan
    for fmt in (1, 2, 3, 4, 5, 6):
        assert orc.quantize(fmt, W, 128).status == orc.NONFINITE


# ------------------------------------------------------------------ dequantization, by hand
def _golden_e2m1_values():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_table.txt")) if l.strip() and not l.startswith("#")]
    return {int(c): float(v) for c, v in rows}


def _h(bits):
    return float(np.uint16(bits).view(np.float16))


# fp16 scales with many significant bits, distinct for s+ and s-
_SP, _SN = 0x3A66, 0x2E1F


def test_dequant_one_fp4_afpq_razer_int8_by_hand(orc):
    """Each format's dequantized value from the golden E2M1 table (or the integer
    code) times a chosen fp16 scale; AFPQ negative codes take s-, positive s+;
    RaZeR's code 0b1000 decodes to the selected special value (+5, -5, +8, -8)."""
    E = _golden_e2m1_values()
    Sp, Sn = _h(_SP), _h(_SN)
    assert Sp != Sn
    for c in range(16):
        assert orc.dequant_one(orc.FP4, c, _SP) == E[c] * Sp, c
        want = E[c] * Sp if E[c] > 0 else E[c] * Sn
        assert orc.dequant_one(orc.AFPQ, c, _SP, _SN) == want, c
        for sel, sv in enumerate([5.0, -5.0, 8.0, -8.0]):
            want = (sv if c == 8 else E[c]) * Sp
            assert orc.dequant_one(orc.RAZER, c, _SP, 0, sel) == want, (c, sel)
        for z in (0, 7, 15):
            assert orc.dequant_one(orc.INT4, c, _SP, 0, z) == (c - z) * Sp, (c, z)
    for q in (-127, -1, 0, 1, 77, 127):
        assert orc.dequant_one(orc.INT8, q & 0xFF, _SN) == q * Sn, q


@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 5])
def test_dequant_matrix_by_hand(orc, fmt):
    """Whole-matrix dequantization with a different scale (and zero / selector)
    for every group, or every row for INT8, against numpy arithmetic on the
    golden E2M1 table: catches a wrong group or row index."""
    rng = np.random.default_rng(40 + fmt)
    N, K, g = 3, 256, 64
    G = 1 if fmt == orc.INT8 else K // g
    E = np.array([_golden_e2m1_values()[c] for c in range(16)])
    s1 = rng.integers(0x2000, 0x3C00, size=N * G).astype(np.uint16)
    s2 = rng.integers(0x2000, 0x3C00, size=N * G).astype(np.uint16)
    z = rng.integers(0, 16 if fmt == orc.INT4 else 4, size=N * G).astype(np.uint8)
    if fmt == orc.INT8:
        codes = rng.integers(-127, 128, size=(N, K)).astype(np.int8).view(np.uint8)
    else:
        codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    q = orc.Quant(fmt, N, K, K if fmt == orc.INT8 else g, codes, s1, s2 if fmt == orc.AFPQ else None,
                  z if fmt in (orc.INT4, orc.RAZER) else None)
    S1 = s1.view(np.float16).astype(np.float64).reshape(N, G)
    S2 = s2.view(np.float16).astype(np.float64).reshape(N, G)
    col = (np.arange(K) // g) if fmt != orc.INT8 else np.zeros(K, int)
    S1k, S2k, Zk = S1[:, col], S2[:, col], z.reshape(N, G)[:, col].astype(np.float64)
    if fmt == orc.INT4:
        want = (codes - Zk) * S1k
    elif fmt == orc.FP4:
        want = E[codes] * S1k
    elif fmt == orc.AFPQ:
        v = E[codes]
        want = np.where(v > 0, v * S1k, v * S2k)
    elif fmt == orc.RAZER:
        sv = np.array([5.0, -5.0, 8.0, -8.0])[z.reshape(N, G)[:, col]]
        want = np.where(codes == 8, sv, E[codes]) * S1k
    else:
        want = codes.view(np.int8).astype(np.float64) * S1k
    assert np.array_equal(orc.dequant(q), want)


# ------------------------------------------------------------------ exact ties (hand-worked)
def _tie_cases():
    for line in open(os.path.join(GOLDEN, "int_ties.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        f = line.split()
        name, fmt, log2s = f[0], f[1], int(f[2])
        w = np.array([float(v) for v in f[3:11]]) * 2.0 ** log2s
        yield name, fmt, w.astype(np.float32), int(f[11], 16), int(f[12]), [int(v) for v in f[13:21]]


def test_int_ties_round_half_to_even(orc):
    """INT4 codes and zero points and INT8 codes at exact .5 ties go to the even
    integer (hand-worked groups in tests/golden/int_ties.txt)."""
    cases = list(_tie_cases())
    assert len(cases) == 3
    for name, fmt, w, sbits, zero, codes in cases:
        if fmt == "int4":
            c, s1, _, z, st = orc.quantize_group(orc.INT4, w)
            assert st == 0 and s1 == sbits and z == zero, name
            assert list(c) == codes, (name, list(c))
        else:
            r = orc.quantize(orc.INT8, w[None, :], w.size)
            assert r.status == 0 and int(r.s1[0]) == sbits, name
            assert list(r.codes.view(np.int8)[0]) == codes, (name, list(r.codes.view(np.int8)[0]))


# ------------------------------------------------------------------ RaZeR: summation order of the error
def _razer_sq_errors(w, sel):
    """Squared errors (binary64) of each weight under RaZeR candidate `sel`,
    codes found by enumerating the whole grid (ties: regular value over the
    special value, then even mantissa)."""
    sv = [5.0, -5.0, 8.0, -8.0][sel]
    am = np.float32(np.max(np.abs(w)))
    s = float(np.float16(am / np.float32(max(6.0, abs(sv)))))
    s = 1.0 if s == 0.0 else s
    out = []
    for x in w:
        v = float(np.float32(x) / np.float32(s))
        grid = [(abs(v - (sv if c == 8 else _e2m1_from_bits(c))), c == 8, c % 2, c) for c in range(16)]
        d = min(t[0] for t in grid)
        ties = [t for t in grid if t[0] == d]
        reg = [t for t in ties if not t[1]]
        c = (min(reg, key=lambda t: t[2])[3] if reg else 8)
        e = float(x) - (sv if c == 8 else _e2m1_from_bits(c)) * s
        out.append(e * e)
    return out


def _tree(t):
    t, width = list(t), 1
    while width < len(t):
        for i in range(0, len(t) - width, 2 * width):
            t[i] = t[i] + t[i + width]
        width *= 2
    return t[0]


def test_razer_selector_uses_tree_order_sum(orc):
    """A group whose candidates +5 and -5 tie under the balanced-tree sum of the
    squared errors but not under a left-to-right sum: the selector is 0 (tree
    tie, smallest selector), not 1 (tests/golden/razer_order_case.txt)."""
    line = [l for l in open(os.path.join(GOLDEN, "razer_order_case.txt")) if l.strip() and not l.startswith("#")][0]
    w = np.array([int(v, 16) for v in line.split()], np.uint32).view(np.float32)
    E = [_razer_sq_errors(w, s) for s in range(4)]
    tree = [_tree(e) for e in E]
    seq = []
    for e in E:                                    # plain left-to-right binary64 sum
        acc = 0.0
        for v in e:
            acc += v
        seq.append(acc)
    assert tree[0] == tree[1] < min(tree[2], tree[3])
    assert seq[1] < seq[0]                         # the case discriminates the two orders
    codes, s1, _, sel, st = orc.quantize_group(orc.RAZER, w)
    assert st == 0 and sel == 0
