"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Every check here compares the oracle against something independent of it:
- values worked by hand (tests/golden/worked_groups.json, each with its citation);
- closed forms, computed exactly in float64 integer arithmetic;
- brute-force searches over a table built from the OCP FP8 definition;
- library routines (torch's float8_e4m3fn cast, numpy/torch float conversions,
  torch's float64 SiLU);
- invariants the quantization must satisfy.
The checks are chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.  CPU only.
"""
import json
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

import oracle
from precision_activation_quantization_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_groups.json")


# --------------------------------------------------------------------------
# Independent reference facts
# --------------------------------------------------------------------------

def e4m3_table() -> np.ndarray:
    """float64 value of each of the 256 E4M3 codes (OCP FP8, 'fn' variant)."""
    vals = np.empty(256, np.float64)
    for c in range(256):
        sign = -1.0 if c & 0x80 else 1.0
        e, m = (c >> 3) & 0xF, c & 7
        if e == 15 and m == 7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


TABLE = e4m3_table()
POS_CODES = np.arange(0, 0x7F)           # 0x00 .. 0x7E: finite, non-negative
POS_VALS = TABLE[POS_CODES]


def brute_e4m3(t) -> np.ndarray:
    """Nearest finite E4M3 code by exhaustive search, ties to the even mantissa.

    |t| is clamped to 448 first; the sign bit is t's sign (so -0 and values that
    round to zero from below give 0x80).
    """
    t = np.asarray(t, np.float64).reshape(-1)
    out = np.empty(t.size, np.uint8)
    for lo in range(0, t.size, 1 << 15):
        a = np.minimum(np.abs(t[lo:lo + (1 << 15)]), 448.0)
        d = np.abs(a[:, None] - POS_VALS[None, :])
        is_min = d == d.min(axis=1, keepdims=True)
        n_min = is_min.sum(axis=1)
        assert n_min.max() <= 2
        even = (POS_CODES % 2 == 0)[None, :]
        pick = np.where((n_min == 1)[:, None], is_min, is_min & even)
        assert (pick.sum(axis=1) == 1).all()
        code = POS_CODES[pick.argmax(axis=1)].astype(np.uint8)
        out[lo:lo + a.size] = code | (np.signbit(t[lo:lo + a.size]).astype(np.uint8) << 7)
    return out


def exact_ue8m0(a) -> np.ndarray:
    """127 + (smallest integer n with 448 * 2^n >= a), exactly, in float64."""
    a = np.asarray(a, np.float32).astype(np.float64).reshape(-1)
    n = np.floor(np.log2(a / 448.0)).astype(np.int64) - 2
    for _ in range(6):
        n = np.where(448.0 * np.exp2(n.astype(np.float64)) >= a, n, n + 1)
    # n is now an upper bound; step down while the predecessor still satisfies it
    for _ in range(6):
        prev_ok = 448.0 * np.exp2((n - 1).astype(np.float64)) >= a
        n = np.where(prev_ok, n - 1, n)
    return (n + 127).astype(np.int64)


def all_bf16_finite() -> np.ndarray:
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    return bits[np.isfinite(vals)], vals[np.isfinite(vals)]


def log_uniform(rng, n, lo_exp, hi_exp, signed=True) -> np.ndarray:
    mag = np.exp2(rng.uniform(lo_exp, hi_exp, n)).astype(np.float32)
    if signed:
        mag *= np.where(rng.random(n) < 0.5, -1, 1).astype(np.float32)
    return mag


# --------------------------------------------------------------------------
# Decoding
# --------------------------------------------------------------------------

def test_decode_bf16_every_pattern_matches_torch():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    got = oracle.decode(bits, "bf16")
    assert np.array_equal(got.view(np.uint32)[np.isfinite(ref)],
                          ref.view(np.uint32)[np.isfinite(ref)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_decode_fp16_every_pattern_matches_numpy():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = oracle.decode(bits, "fp16")
    fin = np.isfinite(ref)
    assert np.array_equal(got.view(np.uint32)[fin], ref.view(np.uint32)[fin])
    assert np.array_equal(np.isinf(got), np.isinf(ref))
    assert np.array_equal(np.isnan(got), np.isnan(ref))


# --------------------------------------------------------------------------
# E4M3 encoder (P-1, P-2)
# --------------------------------------------------------------------------

def test_e4m3_table_matches_torch_and_landmarks():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(lib), np.isnan(TABLE))
    fin = ~np.isnan(TABLE)
    assert np.array_equal(lib[fin], TABLE[fin])
    assert TABLE[0x7E] == 448.0 and np.isnan(TABLE[0x7F]) and np.isnan(TABLE[0xFF])
    assert TABLE[0x01] == 2.0 ** -9 and TABLE[0x08] == 2.0 ** -6
    assert np.nanmax(TABLE) == 448.0


def test_e4m3_round_trip_every_finite_code():
    fin = [c for c in range(256) if not np.isnan(TABLE[c])]
    got = oracle.e4m3_encode(TABLE[fin].astype(np.float32))
    assert list(got) == fin


def test_e4m3_encoder_matches_brute_force():
    rng = np.random.default_rng(11)
    _, bf = all_bf16_finite()
    bf = bf[np.abs(bf) <= 1000.0]
    vals = np.sort(POS_VALS)
    mids = ((vals[1:] + vals[:-1]) / 2.0).astype(np.float32)   # exact in fp32
    mids = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)),
                           np.nextafter(mids, np.float32(-np.inf))])
    mids = np.concatenate([mids, -mids])
    rand = log_uniform(rng, 200_000, -14, 9.5)
    t = np.concatenate([bf, mids, rand, np.float32([0.0, -0.0, 448.0, -448.0, 464.0,
                                                    465.0, 1e30, -1e30])]).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(t), brute_e4m3(t))


def test_e4m3_encoder_matches_torch_cast():
    rng = np.random.default_rng(12)
    t = log_uniform(rng, 1_000_000, -16, 9.2)
    ref = torch.from_numpy(np.clip(t, -448.0, 448.0)).to(torch.float8_e4m3fn)
    assert np.array_equal(oracle.e4m3_encode(t), ref.view(torch.uint8).numpy())


E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def brute_e2m1(t) -> np.ndarray:
    """Nearest OCP E2M1 magnitude by exhaustive search (ties to the even code),
    |t| clamped to 6, sign bit from t."""
    t = np.asarray(t, np.float64).reshape(-1)
    a = np.minimum(np.abs(t), 6.0)
    d = np.abs(a[:, None] - E2M1_MAGS[None, :])
    is_min = d == d.min(axis=1, keepdims=True)
    codes = np.arange(8)
    pick = np.where((is_min.sum(1) == 1)[:, None], is_min, is_min & (codes % 2 == 0)[None, :])
    assert (pick.sum(1) == 1).all()
    return (codes[pick.argmax(1)] | (np.signbit(t).astype(np.int64) << 3)).astype(np.uint8)


def test_e2m1_encoder_matches_brute_force():
    rng = np.random.default_rng(17)
    _, bf = all_bf16_finite()
    bf = bf[np.abs(bf) <= 16.0]
    mids = (E2M1_MAGS[1:] + E2M1_MAGS[:-1]) / 2
    mids = np.concatenate([mids, np.nextafter(mids.astype(np.float32), np.float32(9)),
                           np.nextafter(mids.astype(np.float32), np.float32(-9))])
    t = np.concatenate([bf, mids, -mids, rng.uniform(-8, 8, 100_000),
                        np.float32([0.0, -0.0, 6.0, -6.0, 6.5, 1e9])]).astype(np.float32)
    assert np.array_equal(oracle.e2m1_encode(t), brute_e2m1(t))


def test_ue8m0_with_fmax6_equals_exact_ceiling():
    rng = np.random.default_rng(18)
    _, bf = all_bf16_finite()
    a = np.concatenate([bf[bf >= 1e-10],
                        rng.integers(np.float32(1e-10).view(np.uint32),
                                     np.float32(2.0 ** 120).view(np.uint32), 1_000_000,
                                     dtype=np.uint32).view(np.float32)]).astype(np.float32)
    a64 = a.astype(np.float64)
    n = np.floor(np.log2(a64 / 6.0)).astype(np.int64) - 2
    for _ in range(6):
        n = np.where(6.0 * np.exp2(n.astype(np.float64)) >= a64, n, n + 1)
    for _ in range(6):
        n = np.where(6.0 * np.exp2((n - 1).astype(np.float64)) >= a64, n - 1, n)
    assert np.array_equal(oracle.ue8m0_exponent_fmax(a, 6.0).astype(np.int64), n + 127)


def test_mxfp4_dequant_error_bound_and_nibble_order():
    w = inputs.sweep(M=128, K=1024)
    q, s = oracle.quant(w.x, M=w.M, K=w.K, group=32, out_dtype="e2m1", scale_fmt="ue8m0")
    x = _f32(w.x).reshape(w.M, -1, 32).astype(np.float64)
    lo, hi = q.reshape(w.M, -1) & 0xF, q.reshape(w.M, -1) >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(w.M, -1, 32)      # element 2i low nibble
    vals = E2M1_MAGS[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    sc = np.exp2(s.reshape(w.M, -1, 1).astype(np.float64) - 127)
    err = np.abs(vals * sc - x)
    t = np.abs(x) / sc
    assert (t <= 6.0).all()
    assert (err[t >= 1] <= 0.25 * np.abs(x[t >= 1]) * (1 + 2.0 ** -20)).all()
    assert (err[t < 1] <= 0.25 * np.broadcast_to(sc, x.shape)[t < 1] + 1e-30).all()


# --------------------------------------------------------------------------
# NVFP4: E2M1 codes in blocks of 16, E4M3 block scales, fp32 global scale g
# --------------------------------------------------------------------------

E4M3_MIDS = (np.sort(POS_VALS)[1:] + np.sort(POS_VALS)[:-1]) / 2.0
E2M1_MIDS = (E2M1_MAGS[1:] + E2M1_MAGS[:-1]) / 2.0
NV_SCALES = (1.0, 2.625, 896.0, 0.37109375, 2.0 ** -12, 5000.0)


def _near(v, mids, rel) -> np.ndarray:
    """|v| within `rel` (relative) of one of the rounding midpoints."""
    v = np.abs(np.asarray(v, np.float64)).reshape(-1)
    i = np.clip(np.searchsorted(mids, v), 1, mids.size - 1)
    d = np.minimum(np.abs(v - mids[i - 1]), np.abs(v - mids[i]))
    return d <= rel * np.maximum(v, 1e-300)


def test_e4m3_decode_matches_torch():
    got = oracle.e4m3_decode(np.arange(256)).astype(np.float64)
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    lib = lib.double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(lib))
    fin = ~np.isnan(lib)
    assert np.array_equal(got[fin], lib[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(lib[fin]))


@pytest.mark.parametrize("g", NV_SCALES)
def test_nvfp4_block_scale_is_nearest_e4m3_of_amax_times_g_over_6(g):
    """sf = the E4M3 code nearest to amax * g / 6 (exact arithmetic), saturating
    at 448, except within fp32 rounding of an E4M3 midpoint."""
    rng = np.random.default_rng(31)
    a = np.concatenate([log_uniform(rng, 200_000, -34, 17, signed=False),
                        np.float32([1e-10, 6.0, 3.0, 2688.0])]).astype(np.float32)
    g32 = np.float32(g)
    r = a.astype(np.float64) * np.float64(g32) / 6.0
    near = _near(np.minimum(r, 448.0), E4M3_MIDS, 2.0 ** -21)
    assert near.mean() < 1e-3
    got = oracle.nvfp4_block_scale(a, g32)
    assert np.array_equal(got[~near], brute_e4m3(r)[~near])


@pytest.mark.parametrize("g", NV_SCALES)
def test_nvfp4_multiplier_is_correctly_rounded_g_over_block_scale(g):
    sf = np.arange(0, 0x7F)
    m = oracle.nvfp4_multiplier(sf, np.float32(g)).astype(np.float64)
    assert m[0] == 0.0                                 # a zero block scale zeroes the block
    exact = np.float64(np.float32(g)) / TABLE[sf[1:]]
    ulp = np.spacing(np.abs(m[1:]).astype(np.float32)).astype(np.float64)
    assert (np.abs(m[1:] - exact) <= 0.5 * ulp * (1 + 2.0 ** -20)).all()


def _nvfp4_block(w, g, layout="row"):
    q, s = oracle.quant(w.x, M=w.M, K=w.K, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                        layout=layout, global_scale=g)
    x = _f32(w.x).reshape(w.M, -1, 16).astype(np.float64)
    b = q.reshape(w.M, -1)
    codes = np.stack([b & 0xF, b >> 4], axis=-1).reshape(w.M, -1, 16)   # element 2i low
    return x, codes, s


@pytest.mark.parametrize("g", (2.625, 0.37109375, 5000.0))
def test_nvfp4_codes_are_nearest_e2m1_of_x_times_g_over_block_scale(g):
    """Every code is the E2M1 value nearest to x * g / value(sf) (exact
    arithmetic, saturating at 6); every block scale is nearest to amax * g / 6;
    and dequantized values keep within half an E2M1 step."""
    w = inputs.sweep(M=96, K=1024, seed=33)
    x = _f32(w.x).reshape(96, -1, 16).astype(np.float64)
    x[::7, 3] *= 300.0                                 # outlier blocks
    x[5::11, 9] *= 2.0 ** -40                          # blocks whose scale underflows
    w = w.with_(x=inputs.bf16_bits(x.astype(np.float32)).reshape(1, 96, 1024))
    g32 = np.float64(np.float32(g))
    x, codes, s = _nvfp4_block(w, g)
    sf = s.reshape(96, -1)
    amax = np.maximum(np.abs(x).max(-1), np.float64(np.float32(1e-10)))
    r = amax * g32 / 6.0
    near_s = _near(np.minimum(r, 448.0), E4M3_MIDS, 2.0 ** -21).reshape(sf.shape)
    assert np.array_equal(sf[~near_s], brute_e4m3(r)[~near_s.reshape(-1)])
    d = TABLE[sf][..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = x * g32 / d
        m64 = np.broadcast_to(g32 / d, t.shape)
    # Codes are pinned except near an E2M1 midpoint, where fp32 rounding of the
    # multiplier may decide; an exact tie stays pinned (ties to even) when the
    # multiplier g / value(sf) is exact in fp32.
    ta_c = np.minimum(np.abs(t), 6.0)
    near_c = _near(ta_c, E2M1_MIDS, 2.0 ** -21).reshape(t.shape)
    exact_tie = np.isin(ta_c, E2M1_MIDS) & (m64.astype(np.float32).astype(np.float64) == m64)
    zero_blk = np.broadcast_to(d == 0, t.shape)
    assert zero_blk.any()
    assert np.array_equal(codes[zero_blk], 8 * np.signbit(x[zero_blk]).astype(np.uint8))
    pinned = (~near_c | exact_tie) & ~zero_blk
    assert (~pinned).mean() < 5e-3
    if g == 2.625:                                     # ties do occur: 21/8 over 2^k
        assert exact_tie.sum() > 20
    want = brute_e2m1(t).reshape(t.shape)
    assert np.array_equal(codes[pinned], want[pinned])
    # dequantization: x ~ code * value(sf) / g; a zero block scale zeroes the block
    vals = E2M1_MAGS[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    err = np.abs(vals * d / g32 - x)
    s_x = np.broadcast_to(d / g32, x.shape)
    zero = np.broadcast_to(d == 0, x.shape)
    assert (vals[zero] == 0).all()
    assert (np.abs(x[zero]) <= 6.0 * 2.0 ** -10 / g32).all()
    ta = np.where(zero, 0.0, np.abs(t))
    big, small, sat = (ta >= 1) & (ta <= 6), (ta < 1) & ~zero, ta > 6
    assert (err[big] <= 0.25 * np.abs(x[big]) * (1 + 2.0 ** -20)).all()
    assert (err[small] <= 0.25 * s_x[small] * (1 + 2.0 ** -20)).all()
    assert (err[sat] <= (ta[sat] - 6.0) * s_x[sat] * (1 + 2.0 ** -20)).all()
    if g < 448 * 6 / 300.0 / 8:                        # no block scale saturated
        assert (ta <= 6.0 * (1 + 2.0 ** -4) * (1 + 2.0 ** -20)).all()


def test_nvfp4_zero_block_scale_gives_signed_zero_codes():
    v = np.zeros(48, np.float32)
    v[5] = -0.0                                        # block 0: all zero (amax floored)
    v[16:19] = [2.0 ** -100, -(2.0 ** -100), -(2.0 ** -120)]   # block 1: underflows
    v[32] = 1.0                                        # block 2: ordinary
    w = inputs.Workload("zeros", inputs.bf16_bits(v).reshape(1, 1, 48), M=1, K=48, group=16)
    x, codes, s = _nvfp4_block(w, 1.0)
    assert s.reshape(-1).tolist()[:2] == [0, 0]
    assert codes[0, 0].tolist() == [8 if i == 5 else 0 for i in range(16)]
    assert codes[0, 1, :3].tolist() == [0, 8, 8] and (codes[0, 1, 3:] == 0).all()
    assert s.reshape(-1)[2] == brute_e4m3([1.0 / 6.0])[0]


def test_nvfp4_layouts_and_masking():
    """row, col and 128x4-tiled NVFP4 scales hold the same bytes at their
    positions; masked rows stay untouched; full masks equal flat calls."""
    M, K = 130, 5 * 16                                 # ng = 5: ragged tiles
    x = inputs.bf16_bits(inputs.normal((1, M, K), 34) * 2)
    q_r, s_r = oracle.quant(x, M=M, K=K, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                            layout="row", global_scale=2.625)
    q_c, s_c = oracle.quant(x, M=M, K=K, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                            layout="col", global_scale=2.625)
    q_t, s_t = oracle.quant(x, M=M, K=K, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                            layout="tile128x4", global_scale=2.625)
    assert np.array_equal(q_r, q_c) and np.array_equal(q_r, q_t)
    row = s_r.reshape(M, 5)
    assert np.array_equal(s_c.reshape(5, 132)[:, :M], row.T)
    til = s_t.reshape(-1)
    for (m, g), byte in {(0, 0): 0, (1, 0): 16, (33, 1): 21, (127, 3): 511, (0, 4): 512,
                         (129, 4): 1552}.items():
        assert int(til[byte]) == int(row[m, g]), (m, g, byte)
    for g in (5, 6, 7):                                # padding columns of row 129
        assert til[1024 + 1 * 16 + 512 + g % 4] == 0
    E = 3
    xe = inputs.bf16_bits(inputs.normal((E, 8, 2 * 64), 35))
    mm = np.array([0, 5, 8], np.int32)
    q, s = oracle.quant(xe, E=E, M=8, K=64, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                        layout="row", fused=True, masked_m=mm, global_scale=2.625)
    q, s = q.reshape(E, 8, 32), s.reshape(E, 8, 4)
    for e in range(E):
        assert (q[e, mm[e]:] == 0xA5).all() and (s[e, mm[e]:] == 0xA5).all()
        qf, sf = oracle.quant(xe[e], M=8, K=64, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                              layout="row", fused=True, global_scale=2.625)
        assert np.array_equal(q[e, :mm[e]], qf.reshape(8, 32)[:mm[e]])
        assert np.array_equal(s[e, :mm[e]], sf.reshape(8, 4)[:mm[e]])


def test_int8_encoder_matches_numpy_rint():
    rng = np.random.default_rng(13)
    t = np.concatenate([rng.uniform(-200, 200, 500_000).astype(np.float32),
                        (np.arange(-300, 301) / 2.0).astype(np.float32)])
    ref = np.clip(np.rint(t.astype(np.float64)), -128, 127).astype(np.int8)
    assert np.array_equal(oracle.int8_encode(t), ref)


# --------------------------------------------------------------------------
# Scales (P-8)
# --------------------------------------------------------------------------

def test_ue8m0_bit_algorithm_equals_exact_ceiling():
    rng = np.random.default_rng(14)
    _, bf = all_bf16_finite()
    a_bf = bf[bf >= 1e-10]
    # random fp32 patterns in [1e-10, 2^127]
    lo = np.float32(1e-10).view(np.uint32)
    hi = np.float32(2.0 ** 127).view(np.uint32)
    a_rand = rng.integers(lo, hi, size=10_000_000, dtype=np.uint32).view(np.float32)
    # a near 7 * 2^k, where a/448 sits next to a power of two
    k = np.arange(-30, 120, dtype=np.float64)
    base = (7.0 * np.exp2(k)).astype(np.float32)
    near = [base]
    for _ in range(4):
        near.append(np.nextafter(near[-1], np.float32(np.inf)))
    down = [base]
    for _ in range(4):
        down.append(np.nextafter(down[-1], np.float32(0)))
    a = np.concatenate([a_bf, a_rand] + near + down).astype(np.float32)
    assert np.array_equal(oracle.ue8m0_exponent(a).astype(np.int64), exact_ue8m0(a))


def test_fp32_scale_is_one_ieee_division():
    rng = np.random.default_rng(15)
    a = log_uniform(rng, 500_000, -33, 120, signed=False)
    assert np.array_equal(oracle.scale_fp32(a, "e4m3"), a / np.float32(448.0))
    assert np.array_equal(oracle.scale_fp32(a, "int8"), a / np.float32(127.0))


def test_group_amax_floor_and_sign():
    assert oracle.group_amax(np.zeros(128, np.float32)) == np.float32(1e-10)
    v = np.zeros(128, np.float32)
    v[77] = -3.0
    v[5] = 2.5
    assert oracle.group_amax(v) == 3.0
    v = np.full(128, 1e-12, np.float32)
    assert oracle.group_amax(v) == np.float32(1e-10)


# --------------------------------------------------------------------------
# Hand-worked groups (P-4, P-5, P-6)
# --------------------------------------------------------------------------

def _golden_group(entry) -> np.ndarray:
    v = np.zeros(128, np.float32)
    for i, x in entry["values"].items():
        v[int(i)] = x
    return v


@pytest.mark.parametrize("entry", json.load(open(GOLDEN))["groups"], ids=lambda e: e["name"])
def test_worked_group(entry):
    if "nvfp4" in entry:
        v = np.zeros(entry["K"], np.float32)
        for i, x in entry["values"].items():
            v[int(i)] = x
        nv = entry["nvfp4"]
        q, s = oracle.quant(inputs.bf16_bits(v), M=1, K=entry["K"], group=16, out_dtype="e2m1",
                            scale_fmt="e4m3", layout="row", global_scale=nv["global_scale"])
        assert s.reshape(-1).tolist() == nv["scales"]
        for i, b in nv["bytes"].items():
            assert int(q.reshape(-1)[int(i)]) == b, (entry["name"], i)
        return
    if "e2m1" in entry:
        v = np.zeros(entry["group"], np.float32)
        for i, x in entry["values"].items():
            v[int(i)] = x
        q, s = oracle.quant(inputs.bf16_bits(v), M=1, K=entry["group"], group=entry["group"],
                            out_dtype="e2m1", scale_fmt="ue8m0", layout="row")
        assert int(s.reshape(-1)[0]) == entry["e2m1"]["exponent"]
        for i, b in entry["e2m1"]["bytes"].items():
            assert int(q.reshape(-1)[int(i)]) == b, (entry["name"], i)
        return
    v = _golden_group(entry)
    bits = inputs.bf16_bits(v)
    assert np.array_equal(oracle.decode(bits).view(np.uint32), v.view(np.uint32)), \
        "worked values must be exact bf16"
    if "ue8m0" in entry:
        q, s = oracle.quant(bits, M=1, K=128, group=128, scale_fmt="ue8m0", layout="row")
        assert int(s.reshape(-1)[0]) == entry["ue8m0"]["exponent"]
        for i, c in entry["ue8m0"]["codes"].items():
            assert int(q.reshape(-1)[int(i)]) == c, (entry["name"], i)
    if "fp32" in entry:
        q, s = oracle.quant(bits, M=1, K=128, group=128, scale_fmt="fp32", layout="row")
        if "scale" in entry["fp32"]:
            assert float(s.reshape(-1)[0]) == entry["fp32"]["scale"]
        for i, c in entry["fp32"]["codes"].items():
            assert int(q.reshape(-1)[int(i)]) == c, (entry["name"], i)
    if "int8" in entry:
        q, s = oracle.quant(bits, M=1, K=128, group=128, out_dtype="int8")
        assert float(s.reshape(-1)[0]) == entry["int8"]["scale"]
        for i, c in entry["int8"]["codes"].items():
            assert int(q.view(np.int8).reshape(-1)[int(i)]) == c, (entry["name"], i)


# --------------------------------------------------------------------------
# Exhaustive bf16 sweep in a carrier group (P-3)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("carrier", [448.0, 448.0 * 2 ** -20, 448.0 * 2 ** 20, 1.0,
                                     3.140625, 1e-10])
def test_every_bf16_value_in_a_carrier_group(carrier):
    bits, vals = all_bf16_finite()
    n = bits.size
    # the carrier as the bf16 value it becomes
    A = float(torch.tensor([carrier]).to(torch.bfloat16).float()[0])
    x = np.full((n, 128), A, np.float32)
    x[:, 0] = vals
    xb = inputs.bf16_bits(x)
    amax = np.maximum(np.maximum(np.abs(vals), np.float32(A)), np.float32(1e-10))

    q, s = oracle.quant(xb, M=n, K=128, group=128, scale_fmt="ue8m0", layout="row")
    e = exact_ue8m0(amax)
    assert np.array_equal(s.reshape(-1).astype(np.int64), e)
    scale = np.exp2((e - 127).astype(np.float64))
    q = q.reshape(n, 128)
    assert np.array_equal(q[:, 0], brute_e4m3(vals.astype(np.float64) / scale))
    assert np.array_equal(q[:, 1], brute_e4m3(np.float64(A) / scale))

    q, s = oracle.quant(xb, M=n, K=128, group=128, scale_fmt="fp32", layout="row")
    sf = amax / np.float32(448.0)
    assert np.array_equal(s.reshape(-1), sf)
    q = q.reshape(n, 128)
    assert np.array_equal(q[:, 0], brute_e4m3(vals / sf))
    assert np.array_equal(q[:, 1], brute_e4m3(np.float32(A) / sf))

    q, s = oracle.quant(xb, M=n, K=128, group=128, out_dtype="int8", layout="row")
    si = amax / np.float32(127.0)
    assert np.array_equal(s.reshape(-1), si)
    ref = np.clip(np.rint((vals / si).astype(np.float64)), -128, 127).astype(np.int8)
    assert np.array_equal(q.view(np.int8).reshape(n, 128)[:, 0], ref)


# --------------------------------------------------------------------------
# Invariant (P-7) and the whole path against library primitives
# --------------------------------------------------------------------------

def _f32(bits, in_dtype="bf16"):
    return oracle.decode(bits, in_dtype)


@pytest.mark.parametrize("scale_fmt", ["fp32", "ue8m0"])
def test_dequant_error_bound(scale_fmt):
    w = inputs.flat_hidden(M=256, K=7168)
    q, s = oracle.quant(w.x, M=w.M, K=w.K, group=128, scale_fmt=scale_fmt, layout="row")
    x = _f32(w.x).reshape(w.M, w.K // 128, 128).astype(np.float64)
    if scale_fmt == "ue8m0":
        sc = np.exp2(s.reshape(w.M, -1, 1).astype(np.float64) - 127)
    else:
        sc = s.reshape(w.M, -1, 1).astype(np.float64)
    deq = TABLE[q.reshape(w.M, -1, 128)] * sc
    err = np.abs(deq - x)
    t = np.abs(x) / sc
    normal = t >= 2.0 ** -6
    assert (err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 2.0 ** -20)).all()
    assert (err[~normal] <= 2.0 ** -10 * np.broadcast_to(sc, x.shape)[~normal]
            * (1 + 2.0 ** -20)).all()


def test_int8_dequant_error_bound():
    w = inputs.sweep(M=512, K=4096, out_dtype="int8", group=64)
    q, s = oracle.quant(w.x, M=w.M, K=w.K, group=64, out_dtype="int8")
    x = _f32(w.x).reshape(w.M, -1, 64).astype(np.float64)
    sc = s.reshape(w.M, -1, 1).astype(np.float64)
    err = np.abs(q.view(np.int8).reshape(w.M, -1, 64) * sc - x)
    # half a code step, plus the fp32 rounding of t = x/s (half an ulp of |t| < 128)
    assert (err <= sc * (0.5 + 2.0 ** -18)).all()
    assert q.view(np.int8).max() == 127 or q.view(np.int8).min() == -127


@pytest.mark.parametrize("in_dtype,group", [("bf16", 128), ("fp16", 64), ("bf16", 32),
                                            ("bf16", 1024), ("fp16", 1024)])
def test_whole_path_matches_torch_composition(in_dtype, group):
    """fp32-scale E4M3 path against torch primitives (amax, fp32 division, fp8 cast)."""
    w = inputs.sweep(M=64, K=1024, in_dtype=in_dtype, group=group)
    q, s = oracle.quant(w.x, M=w.M, K=w.K, group=group, in_dtype=in_dtype)
    dt = torch.float16 if in_dtype == "fp16" else torch.bfloat16
    x = torch.from_numpy(w.x.reshape(w.M, w.K).view(np.int16)).view(dt).float()
    xg = x.view(w.M, -1, group)
    amax = xg.abs().amax(-1, keepdim=True).clamp_min(1e-10)
    sc = amax / 448.0
    ref = (xg / sc).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    assert np.array_equal(s.reshape(w.M, -1), sc.squeeze(-1).numpy())
    assert np.array_equal(q.reshape(w.M, -1, group), ref.numpy())


# --------------------------------------------------------------------------
# Fused SiLU-and-mul (P-9)
# --------------------------------------------------------------------------

def test_silu_mul_matches_torch_float64():
    rng = np.random.default_rng(16)
    g = np.concatenate([rng.standard_normal(400_000).astype(np.float32) * 3,
                        np.float32([0.0, -0.0, 30.0, -30.0, 88.0, -88.0, 100.0, -100.0,
                                    1e-30, -1e-30])])
    u = rng.standard_normal(g.size).astype(np.float32)
    ref = (torch.nn.functional.silu(torch.from_numpy(g).double())
           * torch.from_numpy(u).double()).float().numpy()
    got = oracle.silu_mul(g, u)
    ulp = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1
    assert (ulp == 0).mean() > 0.99999


def test_silu_mul_is_correctly_rounded_against_long_double():
    """P-9 in its stated form: silu(g) * u evaluated independently, in 80-bit
    long double and through sigmoid(g) = exp(-log1p(exp(-g))), then rounded once
    to fp32.  The oracle (double, one rounding) must give exactly that value,
    signed zeros and subnormal results included, except where the exact product
    lies within 2^-40 relative of an fp32 rounding midpoint (double's own error,
    about 2^-50, could cross it there)."""
    assert np.finfo(np.longdouble).nmant >= 63, "needs x87 extended long double"
    rng = np.random.default_rng(61)
    g = np.concatenate([rng.standard_normal(200_000).astype(np.float32) * 4,
                        (rng.standard_normal(50_000) * 40).astype(np.float32),
                        np.float32([0.0, -0.0, 1e-30, -1e-30, 30.0, -30.0, 88.0, -88.0,
                                    100.0, -100.0])])
    u = rng.standard_normal(g.size).astype(np.float32)
    u[-10:] = np.float32([1.0, 1.0, 2.0, -0.5, 1.0, 1.0, -3.0, 1.0, 0.25, -1.0])
    gl, ul = g.astype(np.longdouble), u.astype(np.longdouble)
    exact = gl * np.exp(-np.log1p(np.exp(-gl))) * ul
    want = exact.astype(np.float32)
    got = oracle.silu_mul(g, u)
    up = np.nextafter(want, np.float32(np.inf)).astype(np.longdouble)
    dn = np.nextafter(want, np.float32(-np.inf)).astype(np.longdouble)
    w = want.astype(np.longdouble)
    gap = np.minimum(np.abs(exact - (w + up) / 2), np.abs(exact - (w + dn) / 2))
    with np.errstate(divide="ignore", invalid="ignore"):
        near_tie = (exact != 0) & (gap / np.abs(exact) < np.longdouble(2.0) ** -40)
    assert near_tie.mean() < 1e-3
    same = got.view(np.int32) == want.view(np.int32)
    assert same[~near_tie].all(), f"{int((~same & ~near_tie).sum())} results not correctly rounded"
    # silu(+0) * 1 = +0 and silu(-0) * 1 = -0: the bit comparison above covered both signs
    assert want[-10] == 0 and not np.signbit(want[-10]) and np.signbit(want[-9])


def test_fused_gate_is_first_half():
    """silu(gate) * up with gate = columns [0, K), up = columns [K, 2K)."""
    K = 128
    x = np.zeros((1, 2 * K), np.float32)
    x[0, :K] = 2.0           # gate
    x[0, K:] = 1.0           # up
    x[0, 3] = -1.0           # a negative gate entry
    q, s = oracle.quant(inputs.bf16_bits(x), M=1, K=K, group=128, fused=True,
                        scale_fmt="fp32")
    silu2 = 2.0 / (1.0 + np.exp(-2.0))
    silu_m1 = -1.0 / (1.0 + np.exp(1.0))
    assert np.isclose(float(s.reshape(-1)[0]), silu2 / 448.0, rtol=1e-6)
    assert int(q.reshape(-1)[0]) == 0x7E
    assert int(q.reshape(-1)[3]) == int(brute_e4m3([silu_m1 / (silu2 / 448.0)])[0])
    # swapping the halves changes the result, so the order is observable
    xs = np.concatenate([x[:, K:], x[:, :K]], axis=1)
    q2, s2 = oracle.quant(inputs.bf16_bits(xs), M=1, K=K, group=128, fused=True,
                          scale_fmt="fp32")
    assert not np.array_equal(s, s2)


@pytest.mark.parametrize("in_dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("fmt", [
    dict(group=128, out_dtype="e4m3", scale_fmt="ue8m0", layout="col"),
    dict(group=64, out_dtype="int8", scale_fmt="fp32", layout="row"),
    dict(group=32, out_dtype="e2m1", scale_fmt="ue8m0", layout="tile128x4"),
    dict(group=16, out_dtype="e2m1", scale_fmt="e4m3", layout="row", global_scale=2.625),
], ids=["e4m3_ue8m0", "int8_fp32", "mxfp4", "nvfp4"])
def test_fused_equals_plain_where_silu_is_the_identity(fmt, in_dtype):
    """For gate >= 32, e^-gate < 2^-46, so silu(gate) = gate / (1 + e^-gate)
    rounds to gate in fp32 and the fused value is gate * up.  With gates that
    are powers of two that product is exact in the input type, so the fused
    call must give the plain call's bytes on the products, in every format."""
    M, K = 6, 256
    rng = np.random.default_rng(81)
    gate = np.exp2(rng.integers(5, 9, (M, K))).astype(np.float32)        # 32 .. 256
    up_bits = inputs.to_bits(inputs.normal((M, K), 82), in_dtype)
    up = oracle.decode(up_bits, in_dtype)
    prod_bits = inputs.to_bits(gate * up, in_dtype)
    assert np.array_equal(oracle.decode(prod_bits, in_dtype), gate * up)  # exact products
    fused_x = np.concatenate([inputs.to_bits(gate, in_dtype), up_bits], axis=1)
    qf, sf = oracle.quant(fused_x.reshape(1, M, 2 * K), M=M, K=K, in_dtype=in_dtype,
                          fused=True, **fmt)
    qp, sp = oracle.quant(prod_bits.reshape(1, M, K), M=M, K=K, in_dtype=in_dtype, **fmt)
    assert np.array_equal(qf, qp) and np.array_equal(sf, sp)


# --------------------------------------------------------------------------
# Layouts and masked dispatch (P-10)
# --------------------------------------------------------------------------

def test_scale_layouts_are_one_table():
    """row, col and packed hold the same exponents at their stated positions."""
    M, K, G = 6, 5 * 128, 128            # ng = 5: a partial packed word; M_pad = 8
    x = inputs.bf16_bits(inputs.normal((1, M, K), 21) * 10)
    q_r, s_r = oracle.quant(x, M=M, K=K, group=G, scale_fmt="ue8m0", layout="row")
    q_c, s_c = oracle.quant(x, M=M, K=K, group=G, scale_fmt="ue8m0", layout="col")
    q_p, s_p = oracle.quant(x, M=M, K=K, group=G, scale_fmt="ue8m0", layout="packed")
    assert np.array_equal(q_r, q_c) and np.array_equal(q_r, q_p)
    row = s_r.reshape(M, 5)
    col = s_c.reshape(5, 8)
    assert np.array_equal(col[:, :M], row.T)
    assert (col[:, M:] == 0xA5).all()                     # padding rows untouched
    byts = s_p.reshape(2, 8).astype(np.int64)
    for j in range(2):
        for m in range(M):
            w = int(byts[j, m]) & 0xFFFFFFFF
            for b in range(4):
                g = 4 * j + b
                want = int(row[m, g]) if g < 5 else 0
                assert (w >> (8 * b)) & 0xFF == want
    assert (s_p.reshape(2, 8)[:, M:].view(np.uint32) == 0xA5A5A5A5).all()
    # direct check of the row-major table against the exact ceiling
    amax = np.maximum(np.abs(oracle.decode(x).reshape(M, 5, G)).max(-1), np.float32(1e-10))
    assert np.array_equal(row.astype(np.int64), exact_ue8m0(amax).reshape(M, 5))
    q_f, s_f = oracle.quant(x, M=M, K=K, group=G, scale_fmt="fp32", layout="col")
    q_g, s_g = oracle.quant(x, M=M, K=K, group=G, scale_fmt="fp32", layout="row")
    assert np.array_equal(s_f.reshape(5, 8)[:, :M], s_g.reshape(M, 5).T)


def test_tile128x4_layout_positions():
    """The 128x4 tiled UE8M0 layout (MXFP8 producer): bytes at hand-derived
    positions, padding columns 0, padding rows untouched."""
    M, K, G = 130, 5 * 32, 32            # 2 row tiles (ragged), ng = 5 -> 2 column tiles
    x = inputs.bf16_bits(inputs.normal((1, M, K), 24) * 3)
    _, row = oracle.quant(x, M=M, K=K, group=G, scale_fmt="ue8m0", layout="row")
    _, til = oracle.quant(x, M=M, K=K, group=G, scale_fmt="ue8m0", layout="tile128x4")
    row = row.reshape(M, 5)
    til = til.reshape(-1)
    assert til.size == 2 * 2 * 512
    # (m, g) -> byte, worked by hand: tile = (m // 128) * 2 + g // 4, then
    # (m % 32) * 16 + ((m % 128) // 32) * 4 + g % 4 inside the tile
    for (m, g), byte in {(0, 0): 0, (1, 0): 16, (32, 0): 4, (33, 1): 21, (127, 3): 511,
                         (0, 4): 512, (128, 0): 1024, (129, 4): 1552, (129, 0): 1040}.items():
        assert int(til[byte]) == int(row[m, g]), (m, g, byte)
    # padding columns (g = 5..7) of quantized rows are 0; padding rows untouched
    for m in (0, 77, 129):
        for g in (5, 6, 7):
            tile = (m // 128) * 2 + g // 4
            byte = tile * 512 + (m % 32) * 16 + ((m % 128) // 32) * 4 + g % 4
            assert til[byte] == 0
    assert til[1024 + 2 * 16] == 0xA5                        # row 130: a padding row
    # every quantized exponent appears once
    assert sorted(til[til != 0xA5].tolist()) == sorted(row.reshape(-1).tolist() + [0] * (3 * M))


def test_masked_rows_untouched_and_full_mask_equals_flat():
    E, M, K = 3, 8, 256
    x = inputs.bf16_bits(inputs.normal((E, M, 2 * K), 22))
    mm = np.array([0, 5, 8], np.int32)
    q, s = oracle.quant(x, E=E, M=M, K=K, group=128, fused=True, scale_fmt="ue8m0",
                        layout="col", masked_m=mm)
    q = q.reshape(E, M, K)
    s = s.reshape(E, 2, M)
    for e in range(E):
        assert (q[e, mm[e]:] == 0xA5).all()
        assert (s[e, :, mm[e]:] == 0xA5).all()
        qf, sf = oracle.quant(x[e], M=M, K=K, group=128, fused=True, scale_fmt="ue8m0",
                              layout="col")
        assert np.array_equal(q[e, :mm[e]], qf.reshape(M, K)[:mm[e]])
        assert np.array_equal(s[e, :, :mm[e]], sf.reshape(2, M)[:, :mm[e]])
    # out-of-range counts are clamped to [0, M]
    q2, _ = oracle.quant(x, E=E, M=M, K=K, group=128, fused=True, scale_fmt="ue8m0",
                         layout="col", masked_m=np.array([-4, 5, 99], np.int32))
    assert np.array_equal(q2, q.reshape(q2.shape))


@pytest.mark.parametrize("fmt,layout,elem", [
    (dict(group=128, scale_fmt="ue8m0"), "col", 1),
    (dict(group=128, scale_fmt="fp32"), "col", 4),
    (dict(group=32, scale_fmt="ue8m0"), "packed", 4),
    (dict(group=16, out_dtype="e2m1", scale_fmt="e4m3", global_scale=2.625), "col", 1),
], ids=["ue8m0_col", "fp32_col", "packed", "nvfp4_col"])
def test_masked_planes_are_padded_like_flat_ones(fmt, layout, elem):
    """With M = 6 rows per expert the column-major and packed planes are
    ceil4(6) = 8 rows tall, so expert e's plane starts at e times the
    one-expert plane size, and holds what a flat call on that expert writes
    for its live rows; padding rows and masked rows keep the sentinel."""
    E, M, K = 3, 6, 256
    x = inputs.bf16_bits(inputs.normal((E, M, K), 23))
    mm = np.array([6, 3, 0], np.int32)
    _, s = oracle.quant(x, E=E, M=M, K=K, layout=layout, masked_m=mm, **fmt)
    s = s.view(np.uint8).reshape(E, -1)
    ng = K // fmt["group"]
    plane = (ng if layout == "col" else (ng + 3) // 4) * 8 * (elem if layout == "col" else 4)
    assert s.shape[1] == plane
    row = (np.arange(plane) // elem) % 8 if layout == "col" else (np.arange(plane) // 4) % 8
    for e in range(E):
        _, sf = oracle.quant(x[e], M=M, K=K, layout=layout, **fmt)
        sf = sf.view(np.uint8).reshape(-1)
        live = row < mm[e]
        assert np.array_equal(s[e, live], sf[live])
        assert (s[e, ~live] == 0xA5).all()
        assert (sf[row >= M] == 0xA5).all()            # a flat call skips padding rows too


@pytest.mark.parametrize("fmt", [
    dict(group=32, out_dtype="e2m1", scale_fmt="ue8m0"),
    dict(group=128, scale_fmt="ue8m0"),
    dict(group=16, out_dtype="e2m1", scale_fmt="e4m3", global_scale=2.625),
], ids=["mxfp4", "e4m3_ue8m0", "nvfp4"])
def test_masked_tiled_planes_hold_whole_tiles(fmt):
    """128x4-tiled scales of 130 rows take two 128-row tiles per column of
    tiles, so expert e's plane starts at e * 2 * ceil(ng/4) * 512 bytes: a
    fully live expert's plane equals a flat call's, an empty one is untouched."""
    E, M, K = 3, 130, 640
    x = inputs.bf16_bits(inputs.normal((E, M, K), 24))
    mm = np.array([M, 0, M], np.int32)
    _, s = oracle.quant(x, E=E, M=M, K=K, layout="tile128x4", masked_m=mm, **fmt)
    ng = K // fmt["group"]
    plane = 2 * ((ng + 3) // 4) * 512
    s = s.view(np.uint8).reshape(-1)
    assert s.size == E * plane
    s = s.reshape(E, plane)
    for e in (0, 2):
        _, sf = oracle.quant(x[e], M=M, K=K, layout="tile128x4", **fmt)
        assert np.array_equal(s[e], sf.view(np.uint8).reshape(-1))
    assert (s[1] == 0xA5).all()


# --------------------------------------------------------------------------
# Grouped-contiguous (varlen) dispatch: packed tokens in per-expert segments
# --------------------------------------------------------------------------

# (seg_indptr, seg_lens, M) -> token rows, each worked by hand from the rule:
# segment e spans [indptr[e], indptr[e+1]) clamped into [0, M] (end >= start),
# and its first lens[e] rows, clamped into the segment, are tokens.
VARLEN_MASKS = [
    # DeepGEMM-style: segments padded to 4 rows; 3, 0, 8 (of 9 asked) and 4 tokens
    (([0, 4, 4, 12, 16], [3, 0, 9, 4], 16), [0, 1, 2] + list(range(4, 12)) + [12, 13, 14, 15]),
    # no lens: every row of every segment is a token (ragged, unpadded)
    (([0, 3, 5, 9], None, 10), list(range(9))),
    # a negative count, a start below 0, an end past M
    (([-2, 2, 6, 40], [5, -1, 9], 8), [0, 1, 6, 7]),
    # a decreasing offset leaves an empty segment; the next starts at its own offset
    (([0, 6, 3, 8], [2, 4, 3], 8), [0, 1, 3, 4, 5]),
    # segments need not start at row 0 or cover every row
    (([5, 7, 7], [2, 9], 9), [5, 6]),
]


@pytest.mark.parametrize("case,rows", VARLEN_MASKS, ids=[str(i) for i in range(len(VARLEN_MASKS))])
def test_varlen_token_rows_by_hand(case, rows):
    indptr, lens, M = case
    live = oracle.varlen_rows(np.array(indptr, np.int32),
                              None if lens is None else np.array(lens, np.int32), M)
    assert sorted(np.flatnonzero(live).tolist()) == rows


def _varlen_planes(row, live, layout, plane_bytes):
    """The bytes one scale plane of M rows must hold when only the rows with
    live[m] are quantized: the row-major byte table ``row`` [M, ng] at each
    layout's defined position for those rows (padding groups 0), the sentinel
    everywhere else."""
    M, ng = row.shape
    mpad, nw = (M + 3) // 4 * 4, (ng + 3) // 4
    want = np.full(plane_bytes, 0xA5, np.uint8)
    for m in np.flatnonzero(live):
        for g in range(ng if layout in ("row", "col") else 4 * nw):
            v = row[m, g] if g < ng else 0
            if layout == "row":
                want[m * ng + g] = v
            elif layout == "col":
                want[g * mpad + m] = v
            elif layout == "packed":
                want[((g // 4) * mpad + m) * 4 + g % 4] = v
            else:
                r = m % 128
                want[((m // 128) * nw + g // 4) * 512 + (r % 32) * 16 + (r // 32) * 4 + g % 4] = v
    return want


@st.composite
def _varlen_case(draw):
    E = draw(st.integers(1, 5))
    caps = draw(st.lists(st.sampled_from([0, 1, 3, 4, 8, 128]), min_size=E, max_size=E))
    indptr = np.concatenate([[0], np.cumsum(caps)]).astype(np.int32)
    M = int(indptr[-1]) + draw(st.sampled_from([0, 1, 5]))        # trailing rows in no segment
    lens = (np.array([draw(st.integers(-1, c + 2)) for c in caps], np.int32)
            if draw(st.booleans()) else None)
    G = draw(st.sampled_from([32, 64, 128]))
    ng = draw(st.integers(1, 6))
    return indptr, lens, M, G, ng, draw(st.sampled_from(["bf16", "fp16"])), draw(st.integers(0, 999))


@settings(max_examples=50, deadline=None)
@given(_varlen_case(), st.booleans())
def test_varlen_token_rows_are_the_flat_call_rows(case, fused):
    """A varlen call writes, for each token row, exactly the codes and scales a
    flat call over all M packed rows writes for that row (same row of codes,
    same row of one scale plane of M rows, every layout), and leaves every
    other row's codes and scale cells untouched."""
    indptr, lens, M, G, ng, in_dtype, seed = case
    K = ng * G
    x = inputs.to_bits(inputs.normal((1, M, 2 * K if fused else K), seed) * 4, in_dtype)
    live = oracle.varlen_rows(indptr, lens, M)
    kw = dict(M=M, K=K, group=G, in_dtype=in_dtype, fused=fused)
    for fmt, layouts in (("ue8m0", ("row", "col", "packed", "tile128x4")), ("fp32", ("row", "col"))):
        q_flat, s_flat = oracle.quant(x, scale_fmt=fmt, layout="row", **kw)
        q_flat = q_flat.reshape(M, K)
        for layout in layouts:
            q, s = oracle.quant_varlen(x, seg_indptr=indptr, seg_lens=lens, scale_fmt=fmt,
                                       layout=layout, **kw)
            q = q.reshape(M, K)
            assert np.array_equal(q[live], q_flat[live])
            assert (q[~live] == 0xA5).all()
            if fmt == "ue8m0":
                want = _varlen_planes(s_flat.reshape(M, ng), live, layout, s.nbytes)
                assert np.array_equal(s.view(np.uint8).reshape(-1), want), layout
            else:
                f = s.view(np.uint32).reshape(-1)
                ref = s_flat.view(np.uint32).reshape(M, ng)
                mpad = (M + 3) // 4 * 4
                idx = (np.arange(M)[:, None] * ng + np.arange(ng)[None, :] if layout == "row"
                       else np.arange(ng)[None, :] * mpad + np.arange(M)[:, None])
                assert np.array_equal(f[idx[live]], ref[live])
                mask = np.ones(f.size, bool)
                mask[idx[live].reshape(-1)] = False
                assert (f[mask] == 0xA5A5A5A5).all()


@settings(max_examples=25, deadline=None)
@given(_varlen_case(), st.sampled_from([1.0, 2.625]), st.sampled_from(["row", "col", "tile128x4"]))
def test_varlen_nvfp4_token_rows_are_the_flat_call_rows(case, g, layout):
    """The same property for NVFP4 (blocks of 16, E4M3 block scales), fused."""
    indptr, lens, M, _, ng, in_dtype, seed = case
    K = ng * 16
    x = inputs.to_bits(inputs.normal((1, M, 2 * K), seed) * 4, in_dtype)
    live = oracle.varlen_rows(indptr, lens, M)
    kw = dict(M=M, K=K, group=16, in_dtype=in_dtype, out_dtype="e2m1", scale_fmt="e4m3",
              fused=True, global_scale=g)
    q_flat, s_flat = oracle.quant(x, layout="row", **kw)
    q, s = oracle.quant_varlen(x, seg_indptr=indptr, seg_lens=lens, layout=layout, **kw)
    q, q_flat = q.reshape(M, K // 2), q_flat.reshape(M, K // 2)
    assert np.array_equal(q[live], q_flat[live]) and (q[~live] == 0xA5).all()
    want = _varlen_planes(s_flat.reshape(M, ng), live, layout, s.nbytes)
    assert np.array_equal(s.view(np.uint8).reshape(-1), want)


def test_varlen_over_padded_segments_equals_masked_dispatch():
    """Experts padded to M_max rows and laid end to end are the masked layout:
    with indptr = e * M_max and lens = masked_m, the varlen codes and row-major
    scales equal those of masked dispatch over [E, M_max]."""
    E, M, K = 4, 12, 384
    x = inputs.bf16_bits(inputs.normal((E, M, 2 * K), 25))
    mm = np.array([12, 0, 5, 13], np.int32)
    indptr = (np.arange(E + 1) * M).astype(np.int32)
    for fmt in ("ue8m0", "fp32"):
        qm, sm = oracle.quant(x, E=E, M=M, K=K, group=128, fused=True, scale_fmt=fmt,
                              layout="row", masked_m=mm)
        qv, sv = oracle.quant_varlen(x.reshape(E * M, 2 * K), M=E * M, K=K, group=128,
                                     fused=True, scale_fmt=fmt, layout="row",
                                     seg_indptr=indptr, seg_lens=mm)
        assert np.array_equal(qm.reshape(-1), qv.reshape(-1))
        assert np.array_equal(sm.view(np.uint8).reshape(-1), sv.view(np.uint8).reshape(-1))


def test_oracle_rejects_unsupported_combinations():
    x = np.zeros((1, 4, 256), np.uint16)
    with pytest.raises(ValueError):
        oracle.quant(x, M=4, K=256, group=128, out_dtype="int8", scale_fmt="ue8m0")
    with pytest.raises(ValueError):
        oracle.quant(x, M=4, K=256, group=128, scale_fmt="fp32", layout="packed")
    with pytest.raises(ValueError):                       # NVFP4 needs a global scale
        oracle.quant(x, M=4, K=256, group=16, out_dtype="e2m1", scale_fmt="e4m3")
    with pytest.raises(ValueError):
        oracle.quant(x, M=4, K=256, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                     layout="packed", global_scale=1.0)
    with pytest.raises(ValueError):
        oracle.quant(x, M=4, K=256, group=16, out_dtype="e2m1", scale_fmt="e4m3",
                     global_scale=-1.0)
    nan = np.full((1, 4, 256), 0x7FC0, np.uint16)
    with pytest.raises(ValueError):
        oracle.quant(nan, M=4, K=256, group=128)


# --------------------------------------------------------------------------
# The seeded inputs are what their recipes say
# --------------------------------------------------------------------------

def test_inputs_are_deterministic_and_shaped():
    a, b = inputs.tiny(), inputs.tiny()
    assert np.array_equal(a.x, b.x) and a.x.shape == (1, 4, 256)
    w = inputs.flat_hidden(M=256, K=7168)
    x = oracle.decode(w.x).reshape(256, 7168)
    for blk in range(2):
        row, g = 128 * blk + (37 * blk) % 128, blk % 56
        assert (x[row, g * 128:(g + 1) * 128] == 0).all()
    assert (np.abs(x) > 20).mean() > 0.0005           # the x200 outliers exist
    m = inputs.masked(E=4, M_max=64, K=128)
    assert m.x.shape == (4, 64, 256) and m.masked_m.min() >= 0 and m.masked_m.max() <= 64
    d = inputs.masked(E=8, M_max=16, K=128, decode=True)
    assert set(np.unique(d.masked_m)) <= {0, 1} and d.expected_m == 1


# --------------------------------------------------------------------------
# Layout properties at random sizes
# --------------------------------------------------------------------------


@st.composite
def _layout_case(draw):
    E = draw(st.integers(1, 3))
    M = draw(st.sampled_from([0, 1, 2, 3, 4, 5, 7, 9, 130]))
    G = draw(st.sampled_from([32, 64, 128]))
    ng = draw(st.integers(1, 6))
    masked = draw(st.booleans())
    mm = (np.array(draw(st.lists(st.integers(-2, M + 2), min_size=E, max_size=E)), np.int32)
          if masked else None)
    return E, M, G, ng, mm, draw(st.sampled_from(["bf16", "fp16"])), draw(st.integers(0, 999))


def _planes_from_rows(row, live, layout, plane_bytes):
    """The bytes each expert's scale plane must hold: the row-major byte table
    `row` [E, M, ng] placed at the layout's defined positions for the live
    rows (padding groups of those rows 0), the sentinel everywhere else."""
    E, M, ng = row.shape
    mpad, nw = (M + 3) // 4 * 4, (ng + 3) // 4
    want = np.full((E, plane_bytes), 0xA5, np.uint8)
    for e in range(E):
        for m in range(live[e]):
            for g in range(4 * nw if layout != "col" else ng):
                v = row[e, m, g] if g < ng else 0
                if layout == "col":
                    want[e, g * mpad + m] = v
                elif layout == "packed":
                    want[e, ((g // 4) * mpad + m) * 4 + g % 4] = v
                else:
                    r = m % 128
                    want[e, ((m // 128) * nw + g // 4) * 512 + (r % 32) * 16 + (r // 32) * 4
                         + g % 4] = v
    return want


@settings(max_examples=60, deadline=None)
@given(_layout_case())
def test_layouts_hold_one_table_at_random_sizes(case):
    """Every layout holds the row-major table at its defined position: column-
    major S[g][m] over ceil4(M) rows, packed words W[j][m] with group 4j+b in
    byte b, and 128x4 tiles; packed and tiled padding groups of live rows are
    0, and nothing else outside the live rows is written.  Codes do not depend
    on the layout, and masked-off rows keep the sentinel."""
    E, M, G, ng, mm, in_dtype, seed = case
    K = ng * G
    x = inputs.to_bits(inputs.normal((E, M, K), seed) * 4, in_dtype)
    live = np.full(E, M) if mm is None else np.clip(mm, 0, M)
    kw = dict(E=E, M=M, K=K, group=G, in_dtype=in_dtype, masked_m=mm)
    q_row, s_row = oracle.quant(x, scale_fmt="ue8m0", layout="row", **kw)
    q_row = q_row.reshape(E, M, K)
    row = s_row.reshape(E, M, ng)
    for layout in ("col", "packed", "tile128x4"):
        q, s = oracle.quant(x, scale_fmt="ue8m0", layout=layout, **kw)
        assert np.array_equal(q.reshape(E, M, K), q_row)
        s = s.view(np.uint8).reshape(E, -1)
        assert np.array_equal(s, _planes_from_rows(row, live, layout, s.shape[1])), layout
    for e in range(E):
        assert (q_row[e, live[e]:] == 0xA5).all()
        assert (row[e, live[e]:] == 0xA5).all()
    mpad = (M + 3) // 4 * 4
    _, f_row = oracle.quant(x, scale_fmt="fp32", layout="row", **kw)
    _, f_col = oracle.quant(x, scale_fmt="fp32", layout="col", **kw)
    f_row, f_col = f_row.reshape(E, M, ng), f_col.reshape(E, ng, mpad)
    for e in range(E):
        n = live[e]
        assert np.array_equal(f_col[e, :, :n].view(np.uint32), f_row[e, :n].T.view(np.uint32))
        assert (f_col[e, :, n:].view(np.uint32) == 0xA5A5A5A5).all()


@settings(max_examples=40, deadline=None)
@given(_layout_case(), st.sampled_from([1.0, 2.625, 896.0]), st.booleans())
def test_nvfp4_layouts_hold_one_table_at_random_sizes(case, g, fused):
    """The same property for NVFP4's E4M3 block-scale bytes (blocks of 16,
    row, column-major and tiled), which its own loop writes, fused or not."""
    E, M, _, ng, mm, in_dtype, seed = case
    K = ng * 16
    x = inputs.to_bits(inputs.normal((E, M, 2 * K if fused else K), seed) * 4, in_dtype)
    live = np.full(E, M) if mm is None else np.clip(mm, 0, M)
    kw = dict(E=E, M=M, K=K, group=16, in_dtype=in_dtype, out_dtype="e2m1", scale_fmt="e4m3",
              fused=fused, masked_m=mm, global_scale=g)
    q_row, s_row = oracle.quant(x, layout="row", **kw)
    q_row = q_row.reshape(E, M, K // 2)
    row = s_row.reshape(E, M, ng)
    for layout in ("col", "tile128x4"):
        q, s = oracle.quant(x, layout=layout, **kw)
        assert np.array_equal(q.reshape(E, M, K // 2), q_row)
        s = s.view(np.uint8).reshape(E, -1)
        assert np.array_equal(s, _planes_from_rows(row, live, layout, s.shape[1])), layout
    for e in range(E):
        assert (q_row[e, live[e]:] == 0xA5).all()
        assert (row[e, live[e]:] == 0xA5).all()


@settings(max_examples=40, deadline=None)
@given(_layout_case(), st.sampled_from([
    dict(out_dtype="e4m3", scale_fmt="ue8m0", layout="packed"),
    dict(out_dtype="e4m3", scale_fmt="fp32", layout="col"),
    dict(out_dtype="int8", scale_fmt="fp32", layout="row"),
    dict(out_dtype="e2m1", scale_fmt="ue8m0", layout="tile128x4"),
    dict(out_dtype="e2m1", scale_fmt="e4m3", layout="col", global_scale=2.625),
]))
def test_fused_equals_plain_where_silu_is_the_identity_at_random_sizes(case, fmt):
    """The identity of test_fused_equals_plain_where_silu_is_the_identity
    (power-of-two gates >= 32, so silu(gate) * up = gate * up exactly) under
    random experts, rows, masks, layouts and formats."""
    E, M, G, ng, mm, in_dtype, seed = case
    G = 16 if fmt["scale_fmt"] == "e4m3" else G
    K = ng * G
    rng = np.random.default_rng(seed)
    gate = np.exp2(rng.integers(5, 9, (E, M, K))).astype(np.float32)
    up_bits = inputs.to_bits(inputs.normal((E, M, K), seed + 1), in_dtype)
    prod = gate * oracle.decode(up_bits, in_dtype).reshape(E, M, K)
    prod_bits = inputs.to_bits(prod, in_dtype)
    assert np.array_equal(oracle.decode(prod_bits, in_dtype).reshape(E, M, K), prod)
    fused_x = np.concatenate([inputs.to_bits(gate, in_dtype), up_bits], axis=-1)
    kw = dict(E=E, M=M, K=K, group=G, in_dtype=in_dtype, masked_m=mm, **fmt)
    qf, sf = oracle.quant(fused_x, fused=True, **kw)
    qp, sp = oracle.quant(prod_bits, **kw)
    assert np.array_equal(qf, qp) and np.array_equal(sf.view(np.uint8), sp.view(np.uint8))
