"""The GPU parity checker, checked on the CPU.

``check_exact`` and ``check_fused`` decide what "parity" means for the CUDA
path.  Here the oracle's own bytes stand in for the device's: unchanged they
must pass, and each planted deviation that breaks the contract (a code two
steps off, too many one-step flips, a scale byte changed where no rounding
tie allows it, a write to a masked-off row) must fail with the message of the
rule it breaks.  No GPU is used.
"""
import numpy as np
import pytest

import gpu_parity
from gpu_parity import check_exact, check_fused, run_oracle
from test_parity_gpu import make, make_nv

E, M, K = 2, 37, 640
MASK = np.array([37, 5], np.int32)


def _device_returns(monkeypatch, mutate=None):
    """Make run_gpu return the oracle's bytes, changed by mutate(w, q, s)."""
    def fake(w, **kw):
        q, s = run_oracle(w)
        q, s = q.copy(), s.copy()
        if mutate is not None:
            mutate(w, q, s)
        return q, s
    monkeypatch.setattr(gpu_parity, "run_gpu", fake)


def _fp8_fused(layout="col", fmt="ue8m0", out="e4m3"):
    return make(M, K, 128, (out, fmt, layout), fused=True, E=E, seed=5, masked_m=MASK)


def _live_code_index(w, q, lo=0x10, hi=0x70, nth=0):
    """Byte index of the nth code of a live row whose magnitude lies in [lo, hi]."""
    q3 = q.reshape(E, M, K)
    e, m, k = np.nonzero(((q3 & 0x7F) >= lo) & ((q3 & 0x7F) <= hi))
    keep = m < np.clip(MASK, 0, M)[e]
    e, m, k = e[keep][nth], m[keep][nth], k[keep][nth]
    return (e * M + m) * K + k


def test_oracle_bytes_pass_both_checks(monkeypatch):
    _device_returns(monkeypatch)
    check_exact(make(M, K, 64, ("int8", "fp32", "col"), E=E, seed=4, masked_m=MASK))
    stats = check_fused(_fp8_fused())
    assert stats == dict(flip_frac=0.0, scale_flips=0)
    check_fused(make_nv(M, K, 2.625, "row", fused=True, E=E, seed=6, masked_m=MASK))
    check_fused(_fp8_fused("tile128x4", "ue8m0", "e2m1"), max_flip_frac=1e-3)


def test_exact_check_catches_one_changed_byte(monkeypatch):
    w = make(M, K, 64, ("int8", "fp32", "col"), E=E, seed=4, masked_m=MASK)
    _device_returns(monkeypatch, lambda w, q, s: q.__setitem__(123, q[123] ^ 1))
    with pytest.raises(AssertionError, match="codes: 1 of"):
        check_exact(w)
    _device_returns(monkeypatch, lambda w, q, s: s.__setitem__(7, s[7] ^ 0x80))
    with pytest.raises(AssertionError, match="scales: 1 of"):
        check_exact(w)


def test_fused_check_catches_a_two_step_code(monkeypatch):
    def two_steps(w, q, s):
        i = _live_code_index(w, q)
        q[i] += 2
    _device_returns(monkeypatch, two_steps)
    with pytest.raises(AssertionError, match="more than one step"):
        check_fused(_fp8_fused())


def _tie_flips(n):
    """Move n codes of live rows to their other E4M3 neighbour, choosing codes
    whose t = y / s lies within 5% of a step of the rounding midpoint: the
    flips a device's few-ulp SiLU may cause, each within the dequant bound."""
    def mutate(w, q, s):
        import oracle
        xf = oracle.decode(w.x, w.in_dtype).reshape(E, M, 2 * K)
        y = oracle.silu_mul(xf[..., :K], xf[..., K:]).astype(np.float64).reshape(E, M, K)
        sc, _ = gpu_parity._scale_planes(w, s)                    # [E, M, ng]
        t = y / np.repeat(sc, w.group, axis=-1)
        q3 = q.reshape(E, M, K)
        c = q3.astype(np.int64)
        live = np.arange(M)[None, :, None] < np.clip(MASK, 0, M)[:, None, None]
        ok = live & (c >= 1) & (c <= 0x7D) & (t > 0)
        v = gpu_parity.E4M3[c]
        other = np.clip(np.where(t > v, c + 1, c - 1), 0, 0x7E)
        vo = gpu_parity.E4M3[other]
        near = ok & (np.abs(t - (v + vo) / 2) <= 0.05 * np.abs(vo - v))
        idx = np.flatnonzero(near)[:n]
        assert idx.size == n
        q3.reshape(-1)[idx] = other.reshape(-1)[idx].astype(np.uint8)
    return mutate


def test_fused_check_counts_one_step_flips(monkeypatch):
    live = int(np.clip(MASK, 0, M).sum()) * K                  # 26 880 elements
    assert 2 / live < 1e-4 < 4 / live
    _device_returns(monkeypatch, _tie_flips(2))                # 7.4e-5 of them
    assert check_fused(_fp8_fused())["flip_frac"] == 2 / live
    _device_returns(monkeypatch, _tie_flips(4))                # 1.5e-4 > 1e-4
    with pytest.raises(AssertionError, match="of codes differ"):
        check_fused(_fp8_fused())


def test_fused_check_bounds_a_flip_away_from_a_tie(monkeypatch):
    """One code moved by a step where no rounding tie explains it breaks the
    dequant bound even though the flip count is within its budget."""
    def one_step(w, q, s):
        q[_live_code_index(w, q, lo=0x38, hi=0x38)] += 1      # 1.0 -> 1.125 at its scale
    _device_returns(monkeypatch, one_step)
    with pytest.raises(AssertionError, match="dequant error"):
        check_fused(_fp8_fused())


def test_fused_check_catches_a_moved_ue8m0_byte(monkeypatch):
    def bump(w, q, s):
        s[3] += 1                            # expert 0, group 0, row 3 (column-major)
    _device_returns(monkeypatch, bump)
    with pytest.raises(AssertionError, match="away from a power of two"):
        check_fused(_fp8_fused())


def _mxfp4_tie_group(up_bits):
    """A fused MXFP4 call (G = 32, row-major UE8M0) whose expert 0, row 0,
    group 0 has every gate 64 (sigmoid(64) is 1 in fp64) and every up the bf16
    value up_bits, so that each of its 32 elements is 64 * up."""
    w = make(M, K, 32, ("e2m1", "ue8m0", "row"), fused=True, E=E, seed=5, masked_m=MASK)
    x = w.x.reshape(E, M, 2 * K)
    x[0, 0, :32] = 0x4280                            # bf16 64.0
    x[0, 0, K:K + 32] = up_bits
    return w


def _rescaled_group(w, q, s):
    """The group quantized as a device whose amax came out one ulp high would:
    its UE8M0 byte one higher and every code E2M1 3 (6 at the halved scale)."""
    assert s[0] == 127 and (q[:16] == 0x77).all()   # oracle: 2^0 and all codes 6
    s[0] += 1
    q[:16] = 0x55


def test_fused_check_allows_an_mxfp4_byte_flip_at_a_power_of_two(monkeypatch):
    """MXFP4 takes the exponent of amax / 6: amax = 6 * 2^0 sits on a power of
    two, so the byte may move by one (with the group's codes rescaled)."""
    w = _mxfp4_tie_group(0x3DC0)                     # up = 0.09375: 64 * up = 6 exactly
    _device_returns(monkeypatch, _rescaled_group)
    assert check_fused(w, max_flip_frac=1e-3)["scale_flips"] == 1


def test_fused_check_rejects_an_mxfp4_byte_flip_away_from_a_power_of_two(monkeypatch):
    w = _mxfp4_tie_group(0x3DCD)                     # up = 0.10009765625: amax / 6 = 1.0677

    def bump(w, q, s):
        s[0] += 1
        q[:16] = 0x55
    _device_returns(monkeypatch, bump)
    with pytest.raises(AssertionError, match="away from a power of two"):
        check_fused(w, max_flip_frac=1e-3)


def test_fused_check_catches_an_fp32_scale_off_by_2_to_minus_10(monkeypatch):
    def scale(w, q, s):
        f = s.view(np.float32)
        f[9] *= np.float32(1 + 2.0 ** -10)
    _device_returns(monkeypatch, scale)
    with pytest.raises(AssertionError, match="fp32 scale off"):
        check_fused(_fp8_fused("row", "fp32"))


def test_fused_check_catches_writes_to_masked_off_rows(monkeypatch):
    dead_row = (1 * M + 20) * K                     # expert 1 keeps only rows 0..4
    _device_returns(monkeypatch, lambda w, q, s: q.__setitem__(dead_row + 3, 0x11))
    with pytest.raises(AssertionError, match="masked-off codes"):
        check_fused(_fp8_fused())
    ng, mpad = K // 128, (M + 3) // 4 * 4
    dead_scale = 1 * ng * mpad + 2 * mpad + 20      # expert 1, group 2, row 20
    _device_returns(monkeypatch, lambda w, q, s: s.__setitem__(dead_scale, 120))
    with pytest.raises(AssertionError, match="untouched scale bytes"):
        check_fused(_fp8_fused())


def test_fused_check_catches_a_moved_nvfp4_block_scale(monkeypatch):
    w = make_nv(M, K, 2.625, "row", fused=True, E=E, seed=6, masked_m=MASK)

    def bump(w, q, s):
        i = int(np.flatnonzero((s >= 0x10) & (s <= 0x70))[0])
        s[i] += 2
    _device_returns(monkeypatch, bump)
    with pytest.raises(AssertionError, match="block scales differ"):
        check_fused(w)


def test_fused_check_catches_a_two_step_e2m1_code(monkeypatch):
    w = _fp8_fused("tile128x4", "ue8m0", "e2m1")

    def two_steps(w, q, s):
        q3 = q.reshape(E, M, K // 2)
        lo = q3 & 0x7                                # magnitude of the even element
        e, m, k = np.nonzero((lo >= 1) & (lo <= 5))
        keep = m < np.clip(MASK, 0, M)[e]
        e, m, k = e[keep][0], m[keep][0], k[keep][0]
        q3[e, m, k] += 2
    _device_returns(monkeypatch, two_steps)
    with pytest.raises(AssertionError, match="more than one step"):
        check_fused(w, max_flip_frac=1e-3)


def test_fused_check_catches_nonzero_packed_padding(monkeypatch):
    """ng = 5 groups leave bytes 1..3 of each row's second packed word as
    padding, which must hold 0."""
    w = _fp8_fused("packed")
    nw, mpad = 2, (M + 3) // 4 * 4

    def pad(w, q, s):
        s[((0 * nw + 1) * mpad + 4) * 4 + 2] = 7    # expert 0, word 1, row 4, byte 2
    _device_returns(monkeypatch, pad)
    with pytest.raises(AssertionError, match="packed padding bytes must be 0"):
        check_fused(w)


def test_fused_check_catches_codes_in_an_nvfp4_zero_block(monkeypatch):
    """A block whose scale code is 0 must dequantize to 0: a nonzero code
    there fails, even though the flip budget would allow one flip."""
    w = make_nv(M, K, 2.625, "row", fused=True, E=E, seed=6, masked_m=MASK)

    def code(w, q, s):
        b = int(np.flatnonzero(s.reshape(E, M, K // 16)[0, :5] == 0)[0])   # a zero block
        m, blk = divmod(b, K // 16)
        q[(m * K + blk * 16) // 2] = 0x01               # code 0.5: one step from 0
    _device_returns(monkeypatch, code)
    with pytest.raises(AssertionError, match="nonzero codes in zero blocks"):
        check_fused(w, max_flip_frac=1e-3)


def _varlen_fused(layout="col", fmt="ue8m0"):
    from test_parity_gpu import make_var
    return make_var([0, 16, 16, 48], [9, 0, 30], 256, 128, ("e4m3", fmt, layout), fused=True,
                    seed=7, M=52)


@pytest.mark.parametrize("layout,fmt", [("col", "ue8m0"), ("packed", "ue8m0"), ("row", "fp32"),
                                        ("tile128x4", "ue8m0")])
def test_varlen_oracle_bytes_pass_and_padding_writes_fail(monkeypatch, layout, fmt):
    """Varlen calls: the oracle's bytes pass both checks; a code written into a
    padding row (row 12 of segment 0), or a scale cell of a row in no segment,
    fails."""
    w = _varlen_fused(layout, fmt)
    _device_returns(monkeypatch)
    assert check_fused(w)["flip_frac"] == 0.0
    check_exact(w.with_(fused=False, x=w.x[..., :256].copy()))
    _device_returns(monkeypatch, lambda w, q, s: q.__setitem__(12 * 256 + 3, 0x11))
    with pytest.raises(AssertionError, match="masked-off codes"):
        check_fused(w)
    ng = 2

    def scale_cell(w, q, s):
        if layout == "row":
            s[(50 * ng) * 4] ^= 1                  # fp32 scale of row 50 (in no segment)
        elif layout == "col":
            s[0 * 52 + 50] ^= 1                    # group 0 of row 50
        elif layout == "packed":
            s[50 * 4] ^= 1                         # word 0 of row 50
        else:
            s[(50 % 32) * 16 + (50 // 32) * 4] ^= 1
    _device_returns(monkeypatch, scale_cell)
    with pytest.raises(AssertionError, match="untouched scale bytes"):
        check_fused(w)
