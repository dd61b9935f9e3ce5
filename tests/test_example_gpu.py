"""The usage example shown to users (the same calls as the README's Python
block, kept here as test code) runs and returns the shapes it states."""
import pytest

pytestmark = pytest.mark.gpu


def test_usage_example_runs():
    import torch
    from precision_activation_quantization_b200 import pqg

    x = torch.randn(8192, 7168, device="cuda", dtype=torch.bfloat16)

    # DeepGEMM-style FP8: G = 128, UE8M0 exponents packed 4 per int32, column-major
    q, s = pqg.quant(x, group=128, scale_fmt="ue8m0", layout="packed")
    assert tuple(q.shape) == (1, 8192, 7168) and q.dtype == torch.float8_e4m3fn
    assert tuple(s.shape) == (1, 56 // 4, 8192) and s.dtype == torch.int32

    # fp32 scales, row-major; INT8 codes; per-token (one scale per row)
    q, s = pqg.quant(x, group=128, scale_fmt="fp32", layout="row")
    assert tuple(s.shape) == (1, 8192, 56) and s.dtype == torch.float32
    q, s = pqg.quant(x, group=128, out_dtype="int8")
    assert q.dtype == torch.int8
    q, s = pqg.quant(x, group=7168)
    assert tuple(s.shape) == (1, 8192, 1)

    # MXFP8 / MXFP4 operands: G = 32, UE8M0 in the 128x4 tiled layout
    q, s = pqg.quant(x, group=32, scale_fmt="ue8m0", layout="tile128x4")
    q4, s4 = pqg.quant(x, group=32, out_dtype="e2m1", scale_fmt="ue8m0", layout="tile128x4")
    assert tuple(s.shape) == (1, 64 * 56 * 512)

    # NVFP4: blocks of 16, E4M3 block scales under a global scale g read on the device
    g = torch.tensor([448 * 6 / x.abs().max().item()], device="cuda")
    q4, sf = pqg.quant(x, group=16, out_dtype="e2m1", scale_fmt="e4m3", layout="tile128x4",
                       global_scale=g)
    assert tuple(q4.shape) == (1, 8192, 3584) and q4.dtype == torch.uint8

    # grouped-contiguous MoE: 3 experts' tokens packed in segments padded to 128 rows
    xp = torch.randn(384, 2 * 2048, device="cuda", dtype=torch.bfloat16)
    indptr = torch.tensor([0, 128, 128, 384], device="cuda", dtype=torch.int32)
    lens = torch.tensor([100, 0, 200], device="cuda", dtype=torch.int32)
    q, s = pqg.quant_varlen(xp, indptr, lens, group=128, scale_fmt="ue8m0", layout="col",
                            fuse_silu_mul=True)
    assert tuple(q.shape) == (384, 2048) and q.dtype == torch.float8_e4m3fn
    assert tuple(s.shape) == (16, 384)

    # fused SiLU-and-mul over [gate | up] rows, masked MoE dispatch
    h = torch.randn(32, 2048, 2 * 2048, device="cuda", dtype=torch.bfloat16)
    masked_m = torch.randint(0, 2049, (32,), device="cuda", dtype=torch.int32)
    q, s = pqg.quant(h, group=128, scale_fmt="ue8m0", layout="col", fuse_silu_mul=True,
                     masked_m=masked_m, expected_m=1024)
    torch.cuda.synchronize()
    assert tuple(q.shape) == (32, 2048, 2048)
    assert tuple(s.shape) == (32, 16, 2048)
