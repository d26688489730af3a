"""Decode-time cache maintenance on the GPU, through the C ABI: the MXFP4 quantizer of the
indexer rows (bit-exact against the oracle's OCP MX v1.0 encoder on FP32 and BF16 input,
including every rounding tie, zero blocks, saturation and negative values that round to
zero), and the window ring buffer against the linear window (the same decode batch
attended through a ring of W rows per sequence and through linear rows gives the same
result; the harness checks both against the oracle)."""
import numpy as np
import pytest
import torch

import long_context_sparse_softmax_b200 as lc
from long_context_sparse_softmax_b200 import workloads as wl
from oracle import lc_oracle as O
from tests.gpu_checks import check_decode

pytestmark = pytest.mark.gpu


def _quantize(x: torch.Tensor, fmt: int):
    n, d = x.shape
    codes = torch.empty(n, d // 2, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, d // 32, dtype=torch.uint8, device="cuda")
    lc.lc_mxfp4_quantize(lc.Mxfp4QuantArgs(n, d, fmt, x.data_ptr(), codes.data_ptr(), scales.data_ptr()))
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def _crafted_rows(rng, n, d):
    v = rng.standard_normal((n, d)) * np.exp2(rng.integers(-20, 20, (n, 1)))
    grid = O.e2m1_to_f64(np.arange(8))
    ties = (grid[:-1] + grid[1:]) / 2
    # rows of exact ties under a block scale of 2^-3 (block max 6 * 2^-3 pins the scale)
    for r in range(0, n, 7):
        t = rng.choice(np.concatenate([ties, -ties, grid, -grid]), d) * 0.125
        t[::32] = 6 * 0.125
        v[r] = t
    v[1, :32] = 0.0                       # a zero block
    v[2, 32:64] = -1e-3                   # small negatives next to a large one: round to zero
    v[2, 32] = 7.9                        # block max just below 8: X = 2^0 ... saturates at 6
    v[3] = -v[3]
    return v


@pytest.mark.parametrize("d", [128, 64, 256])
def test_mxfp4_quantize_f32_bit_exact(d):
    rng = np.random.default_rng(90 + d)
    v = _crafted_rows(rng, 300, d).astype(np.float32)
    codes, scales = _quantize(torch.from_numpy(v).cuda(), lc.LC_FMT_F32)
    ec, es = O.f64_to_mxfp4(v.astype(np.float64))
    assert np.array_equal(scales, es)
    assert np.array_equal(codes, ec), f"{int((codes != ec).sum())} code bytes differ"


def test_mxfp4_quantize_bf16_bit_exact():
    rng = np.random.default_rng(95)
    v = torch.from_numpy(_crafted_rows(rng, 500, 128)).to(torch.bfloat16)
    codes, scales = _quantize(v.view(torch.int16).cuda(), lc.LC_FMT_BF16)
    ec, es = O.f64_to_mxfp4(v.double().numpy())
    assert np.array_equal(scales, es) and np.array_equal(codes, ec)


@pytest.mark.parametrize("ring", [True, False], ids=["ring", "linear"])
def test_decode_window_ring_and_linear(ring):
    """Lengths whose windows wrap around the ring (L mod 128 != 0), one that starts at slot 0
    (L = 1024, two window tiles), sequences shorter than the window."""
    s = wl.shrink(wl.CSA_DECODE, name=f"ring_{ring}", seed=96, seq_lens=(1000, 1024, 70, 4099, 128, 9000),
                  k=128, ring=ring)
    rep = check_decode(s)
    assert rep["attn_e2e_rows_checked"] == 6 * 64


def test_hca_decode_window_ring():
    s = wl.shrink(wl.MIXED_HCA, name="ring_hca", seed=97, seq_lens=(128 * 30 + 77, 1000, 64, 128 * 8))
    check_decode(s)
