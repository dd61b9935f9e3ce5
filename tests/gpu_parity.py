"""Helpers shared by the GPU parity tests: run a workload through the C ABI and
through the oracle, and compare the results.

The kernel's output and scale buffers are filled with a sentinel byte first and
carry a guard band past their end, so that writes to rows the call must not
touch, or writes past the buffer, show up as changed sentinel bytes.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle
from precision_activation_quantization_b200 import pqg

SENTINEL = 0xA5
GUARD = 4096


def _torch_input(w):
    dt = torch.float16 if w.in_dtype == "fp16" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(w.x).view(np.int16)).view(dt).cuda()


def run_gpu(w, *, expected_m=None, stream=None, x_dev=None):
    """Run ``w`` through pqg_quant (pqg_quant_nvfp4 for E4M3 block scales);
    returns (codes uint8 [E*M*K], scale bytes)."""
    x = _torch_input(w) if x_dev is None else x_dev
    n_out = w.E * w.M * (w.K // 2 if w.out_dtype == "e2m1" else w.K)
    nbytes = pqg.pqg_scales_bytes(w.E, w.M, w.K, w.group, pqg.SCALE_FMTS[w.scale_fmt],
                                  pqg.LAYOUTS[w.layout])
    assert nbytes >= 0
    out = torch.full((n_out + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
    sc = torch.full((nbytes + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
    mm = None if w.masked_m is None else torch.from_numpy(np.asarray(w.masked_m, np.int32)).cuda()
    s = stream if stream is not None else torch.cuda.current_stream()
    em = w.expected_m if expected_m is None else expected_m
    if w.seg_indptr is not None:
        ip = torch.from_numpy(np.asarray(w.seg_indptr, np.int32)).cuda()
        ln = None if w.seg_lens is None else torch.from_numpy(np.asarray(w.seg_lens, np.int32)).cuda()
        gsc = (torch.tensor([w.global_scale], dtype=torch.float32, device="cuda")
               if w.scale_fmt == "e4m3" else None)
        st = pqg.pqg_quant_varlen(x.data_ptr(), out.data_ptr(), sc.data_ptr(),
                                  None if gsc is None else gsc.data_ptr(), w.M, w.segments,
                                  w.K, w.group, pqg.IN_DTYPES[w.in_dtype],
                                  pqg.OUT_DTYPES[w.out_dtype], pqg.SCALE_FMTS[w.scale_fmt],
                                  pqg.LAYOUTS[w.layout], int(w.fused), ip.data_ptr(),
                                  None if ln is None else ln.data_ptr(), em, s.cuda_stream)
    elif w.scale_fmt == "e4m3":
        gsc = torch.tensor([w.global_scale], dtype=torch.float32, device="cuda")
        st = pqg.pqg_quant_nvfp4(x.data_ptr(), out.data_ptr(), sc.data_ptr(), gsc.data_ptr(),
                                 w.M, w.E, w.K, pqg.IN_DTYPES[w.in_dtype],
                                 pqg.LAYOUTS[w.layout], int(w.fused),
                                 None if mm is None else mm.data_ptr(), em, s.cuda_stream)
    else:
        st = pqg.pqg_quant(x.data_ptr(), out.data_ptr(), sc.data_ptr(), w.M, w.E, w.K, w.group,
                           pqg.IN_DTYPES[w.in_dtype], pqg.OUT_DTYPES[w.out_dtype],
                           pqg.SCALE_FMTS[w.scale_fmt], pqg.LAYOUTS[w.layout], int(w.fused),
                           None if mm is None else mm.data_ptr(), em, s.cuda_stream)
    assert st == pqg.PQG_OK, pqg.pqg_status_string(st)
    torch.cuda.synchronize()
    out_h, sc_h = out.cpu().numpy(), sc.cpu().numpy()
    assert (out_h[n_out:] == SENTINEL).all(), "codes written past the end of the buffer"
    assert (sc_h[nbytes:] == SENTINEL).all(), "scales written past the end of the buffer"
    return out_h[:n_out], sc_h[:nbytes]


def run_oracle(w):
    """The oracle's (codes uint8 [E*M*K], scale bytes), sentinel-filled like run_gpu."""
    if w.seg_indptr is not None:
        q, s = oracle.quant_varlen(w.x, M=w.M, K=w.K, group=w.group, seg_indptr=w.seg_indptr,
                                   seg_lens=w.seg_lens, in_dtype=w.in_dtype,
                                   out_dtype=w.out_dtype, scale_fmt=w.scale_fmt,
                                   layout=w.layout, fused=w.fused, fill=SENTINEL,
                                   global_scale=w.global_scale)
        return q.reshape(-1), s.view(np.uint8).reshape(-1)
    q, s = oracle.quant(w.x, E=w.E, M=w.M, K=w.K, group=w.group, in_dtype=w.in_dtype,
                        out_dtype=w.out_dtype, scale_fmt=w.scale_fmt, layout=w.layout,
                        fused=w.fused, masked_m=w.masked_m, fill=SENTINEL,
                        global_scale=w.global_scale)
    return q.reshape(-1), s.view(np.uint8).reshape(-1)


def assert_same(gpu, ref, what):
    gpu, ref = np.ravel(gpu), np.ravel(ref)
    if np.array_equal(gpu, ref):
        return
    bad = np.flatnonzero(gpu != ref)
    raise AssertionError(f"{what}: {bad.size} of {ref.size} bytes differ; first at "
                         f"{bad[:8].tolist()} gpu={gpu[bad[:8]].tolist()} "
                         f"oracle={ref[bad[:8]].tolist()}")


def check_exact(w, **kw):
    """Non-fused contract: codes, scales and untouched bytes are bit-identical."""
    gq, gs = run_gpu(w, **kw)
    rq, rs = run_oracle(w)
    assert_same(gq, rq, f"{w.name} codes")
    assert_same(gs, rs, f"{w.name} scales")
    return gq, gs


# --------------------------------------------------------------------------
# The fused tolerance contract
# --------------------------------------------------------------------------

def _e4m3_values() -> np.ndarray:
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).double().numpy()


E4M3 = _e4m3_values()
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0] + [-0.0, -0.5, -1.0, -1.5, -2.0, -3.0,
                                                          -4.0, -6.0])
E2M1_RANK = np.searchsorted(np.sort(np.unique(E2M1)), E2M1)   # code -> position, +-0 merged


def _unpack_e2m1(b: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] 4-bit codes (element 2i in the low nibble)."""
    return np.stack([b & 0xF, b >> 4], axis=-1).reshape(*b.shape[:-1], -1)
_FINITE = np.sort(np.unique(E4M3[~np.isnan(E4M3)]))     # -448 .. 448, one zero
E4M3_RANK = np.searchsorted(_FINITE, np.nan_to_num(E4M3))  # code -> position


def _scale_planes(w, sbytes):
    """Per-group scales as float64 [E, M, ng] from the scale buffer (for NVFP4
    the dequantization factor value(sf) / g), and the matching byte table
    (UE8M0 exponents or E4M3 block-scale codes; None for fp32 scales)."""
    ng, mpad = w.K // w.group, (w.M + 3) // 4 * 4
    if w.scale_fmt != "fp32":
        if w.layout == "tile128x4":
            m = np.arange(w.M)[:, None]
            g = np.arange(ng)[None, :]
            off = (((m // 128) * ((ng + 3) // 4) + g // 4) * 512 + (m % 32) * 16
                   + ((m % 128) // 32) * 4 + g % 4)
            plane = sbytes.reshape(w.E, -1)
            e8 = plane[:, off]
        elif w.layout == "packed":
            words = sbytes.reshape(w.E, (ng + 3) // 4, mpad, 4)
            e8 = words.transpose(0, 2, 1, 3).reshape(w.E, mpad, -1)[:, :w.M, :ng]
        elif w.layout == "col":
            e8 = sbytes.reshape(w.E, ng, mpad)[:, :, :w.M].transpose(0, 2, 1)
        else:
            e8 = sbytes.reshape(w.E, w.M, ng)
        if w.scale_fmt == "e4m3":
            return E4M3[e8] / np.float64(np.float32(w.global_scale)), e8
        return np.exp2(e8.astype(np.float64) - 127.0), e8
    f = sbytes.view(np.float32)
    if w.layout == "col":
        f = f.reshape(w.E, ng, mpad)[:, :, :w.M].transpose(0, 2, 1)
    else:
        f = f.reshape(w.E, w.M, ng)
    return f.astype(np.float64), None


CONTRACT_FLIP_FRAC = 1e-4     # fused codes: one-step flips on at most 1e-4 of elements
SMALL_SAMPLE = 100_000         # below this many elements a looser budget may be passed


def _log_flips(w, flips, n_el, scale_flips, budget):
    """Print the observed flip count, and append it as a JSON line to the file
    named by PQG_FLIP_LOG when that variable is set."""
    rec = dict(workload=w.name, E=int(w.E), M=int(w.M), K=int(w.K), group=int(w.group),
               in_dtype=w.in_dtype, out_dtype=w.out_dtype, scale_fmt=w.scale_fmt,
               layout=w.layout, elements=int(n_el), flips=flips, flip_frac=flips / max(n_el, 1),
               scale_flips=scale_flips, budget=budget)
    print("fused flips", rec)
    path = os.environ.get("PQG_FLIP_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


def check_fused(w, *, max_flip_frac=CONTRACT_FLIP_FRAC, rel_tol=7e-2, **kw):
    """Fused contract: UE8M0 bytes equal unless the oracle's amax/FMAX (448 for
    E4M3, 6 for E2M1) is within 2^-20 of a power of two; fp32 scales within 2^-19 relative; codes equal
    except for at most ``max_flip_frac`` of elements (outside groups whose UE8M0
    exponent flipped), each moving by one step; every element's dequantized
    value within ``rel_tol`` of the oracle's silu(gate)*up."""
    gq, gs = run_gpu(w, **kw)
    rq, rs = run_oracle(w)
    E, M, K, G = w.E, w.M, w.K, w.group
    if w.seg_indptr is not None:                                       # varlen: one plane
        live = oracle.varlen_rows(w.seg_indptr, w.seg_lens, M)[None, :]
    else:
        rows = np.full(E, M) if w.masked_m is None else np.clip(w.masked_m, 0, M)
        live = np.arange(M)[None, :] < rows[:, None]                   # [E, M]

    # untouched rows and padding must be byte-identical (sentinels)
    kb = K // 2 if w.out_dtype == "e2m1" else K
    gq3, rq3 = gq.reshape(E, M, kb), rq.reshape(E, M, kb)
    assert_same(gq3[~live], rq3[~live], f"{w.name} masked-off codes")
    if w.out_dtype == "e2m1":
        gq3, rq3 = _unpack_e2m1(gq3), _unpack_e2m1(rq3)
    g_sc, g_e8 = _scale_planes(w, gs)
    r_sc, r_e8 = _scale_planes(w, rs)
    # scale bytes outside live (row, group) cells must be untouched
    ng, mpad = K // G, (M + 3) // 4 * 4
    idx = np.arange(gs.size)
    if w.layout == "tile128x4":
        plane = (M + 127) // 128 * ((ng + 3) // 4) * 512
        e_of, off = idx // plane, idx % plane
        tile, inner = off // 512, off % 512
        m_of = (tile // ((ng + 3) // 4)) * 128 + ((inner // 4) % 4) * 32 + inner // 16
    elif w.layout == "packed":
        word = idx // 4
        m_of, e_of = word % mpad, word // (((ng + 3) // 4) * mpad)
    else:
        elem = idx // (4 if w.scale_fmt == "fp32" else 1)
        if w.layout == "col":
            m_of, e_of = elem % mpad, elem // (ng * mpad)
        else:
            m_of, e_of = (elem // ng) % M, elem // (M * ng)
    inside = (m_of < M) & live[e_of, np.minimum(m_of, max(M - 1, 0))]
    assert_same(gs[~inside], rs[~inside], f"{w.name} untouched scale bytes")
    if w.layout == "packed":
        j = (idx // 4 // mpad) % ((ng + 3) // 4)
        pad = inside & (4 * j + idx % 4 >= ng)
        assert (gs[pad] == 0).all(), "packed padding bytes must be 0"

    # the oracle's fused values, for the dequant bound and the flip exemption
    import oracle as _o
    xf = _o.decode(w.x, w.in_dtype).reshape(E, M, 2 * K)
    y = _o.silu_mul(xf[..., :K], xf[..., K:]).astype(np.float64)      # [E, M, K]
    yg = y.reshape(E, M, K // G, G)
    amax = np.maximum(np.abs(yg).max(-1), 1e-10)

    g_sc, r_sc = g_sc[live], r_sc[live]                                # [n_live, ng]
    if g_e8 is not None and w.scale_fmt == "e4m3":
        # NVFP4: the block-scale code may move only where amax * g / 6 lies
        # within a few fp32 ulps of an E4M3 rounding midpoint
        g_e8, r_e8 = g_e8[live].astype(np.int64), r_e8[live].astype(np.int64)
        scale_diff = g_e8 != r_e8
        r = np.minimum(amax[live] * np.float64(np.float32(w.global_scale)) / 6.0, 448.0)
        vals = np.sort(np.unique(np.abs(E4M3[~np.isnan(E4M3)])))
        mids = (vals[1:] + vals[:-1]) / 2.0
        dist = np.min(np.abs(r[..., None] / mids - 1.0), axis=-1)
        assert (~scale_diff | (dist < 2.0 ** -18)).all(), \
            f"{w.name}: {int((scale_diff & (dist >= 2.0 ** -18)).sum())} block scales differ"
        assert (np.abs(E4M3_RANK[g_e8] - E4M3_RANK[r_e8]) <= 1).all()
        exempt = scale_diff
    elif g_e8 is not None:
        g_e8, r_e8 = g_e8[live].astype(np.int64), r_e8[live].astype(np.int64)
        scale_diff = g_e8 != r_e8
        # the byte is the exponent of amax / FMAX: 448 for E4M3, 6 for E2M1 (MXFP4)
        r = amax[live] / (6.0 if w.out_dtype == "e2m1" else 448.0)
        near_pow2 = np.abs(r / np.exp2(np.round(np.log2(r))) - 1.0) < 2.0 ** -20
        assert (~scale_diff | near_pow2).all(), \
            f"{w.name}: {int((scale_diff & ~near_pow2).sum())} UE8M0 bytes differ away from a power of two"
        exempt = scale_diff            # an exponent flip rescales the whole group
    else:
        # the device forms silu(gate)*up in fp32 (a few ulps from the oracle's
        # double), so the group absmax, and with it the scale, may move by a
        # few ulps: bound it at 2^-19 relative
        rel = np.abs(g_sc / r_sc - 1.0)
        assert rel.max(initial=0) <= 2.0 ** -19, f"{w.name}: fp32 scale off by {rel.max():.3g}"
        exempt = np.zeros_like(g_sc, dtype=bool)
        scale_diff = rel > 0

    gcodes = gq3[live].reshape(-1, K // G, G)
    rcodes = rq3[live].reshape(-1, K // G, G)
    diff = (gcodes != rcodes) & ~exempt[..., None]
    n_el = gcodes.size
    if w.out_dtype == "int8":
        step = np.abs(gcodes.view(np.int8).astype(np.int64) - rcodes.view(np.int8).astype(np.int64))
    elif w.out_dtype == "e2m1":
        step = np.abs(E2M1_RANK[gcodes].astype(np.int64) - E2M1_RANK[rcodes].astype(np.int64))
    else:
        step = np.abs(E4M3_RANK[gcodes].astype(np.int64) - E4M3_RANK[rcodes].astype(np.int64))
    assert (step[diff] <= 1).all(), f"{w.name}: a code moved by more than one step"
    frac = diff.sum() / max(n_el, 1)
    # The contract allows one-step flips on at most 1e-4 of elements.  A looser
    # budget may be passed for small samples only: under 1e5 elements a single
    # flip at a rounding tie is already 1e-5 or more.  From 1e5 elements up the
    # contract's 1e-4 applies, whatever budget was passed.
    budget = max_flip_frac if n_el < SMALL_SAMPLE else min(max_flip_frac, CONTRACT_FLIP_FRAC)
    _log_flips(w, int(diff.sum()), n_el, int(scale_diff.sum()), budget)
    assert frac <= budget, f"{w.name}: {frac:.2e} of codes differ (> {budget})"

    # dequantized GPU value vs the oracle's y, per element
    vals = (gcodes.view(np.int8).astype(np.float64) if w.out_dtype == "int8"
            else E2M1[gcodes] if w.out_dtype == "e2m1" else E4M3[gcodes])
    deq = vals * g_sc[..., None]
    yl = y[live].reshape(-1, K // G, G)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.abs(yl) / g_sc[..., None]
    err = np.abs(deq - yl)
    if w.out_dtype == "int8":
        assert (err <= (0.5 + 1.0) * g_sc[..., None]).all()
    elif w.out_dtype == "e2m1":
        # one step of E2M1 is at most half the value (normal) or 0.5 * s; an
        # NVFP4 block's largest element may also saturate from up to 6.4 to 6.
        # An NVFP4 block whose scale rounds to zero (amax * g / 6 <= 2^-10)
        # dequantizes to zero.
        zero = np.broadcast_to(g_sc[..., None] == 0, t.shape)
        if zero.any():
            assert w.scale_fmt == "e4m3" and (vals[zero] == 0).all(), \
                f"{w.name}: nonzero codes in zero blocks"
            bound0 = 6.0 * 2.0 ** -10 / np.float64(np.float32(w.global_scale))
            assert (err[zero] <= bound0 * (1 + 2.0 ** -10)).all(), f"{w.name}: zero blocks"
        # An NVFP4 block scale saturated at 448 leaves t above 6: those codes
        # saturate too, and the error is what lies beyond 6 * scale.
        sc_b = np.broadcast_to(g_sc[..., None], t.shape)
        sat = (t > 6.5) & ~zero
        if sat.any():
            assert w.scale_fmt == "e4m3" and (np.abs(vals[sat]) == 6).all()
            assert (err[sat] <= (t[sat] - 6.0) * sc_b[sat] * (1 + 2.0 ** -10)).all()
        big = (t >= 1.0) & ~zero & ~sat
        small = (t < 1.0) & ~zero
        assert (err[big] <= 0.5 * np.abs(yl[big]) + 1e-30).all(), f"{w.name}: dequant error"
        assert (err[small] <= sc_b[small] * 0.75).all()
    else:
        big = t >= 2.0 ** -6
        assert (err[big] <= rel_tol * np.abs(yl[big])).all(), f"{w.name}: dequant error"
        small_bound = np.broadcast_to(g_sc[..., None], t.shape)[~big] * 2.0 ** -9
        assert (err[~big] <= small_bound).all(), f"{w.name}: dequant error near zero"
    return dict(flip_frac=float(frac), scale_flips=int(scale_diff.sum()))
