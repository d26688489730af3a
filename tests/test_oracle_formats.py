"""Pins of the oracle's number-format codecs against published tables and torch's own
casts (an independent implementation), and of the generator's MXFP4 encoder."""
import os

import numpy as np
import pytest
import torch

from oracle import lc_oracle as O
from long_context_sparse_softmax_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                a, b = line.split()
                rows.append((a, float(b)))
    return rows


def test_e4m3_table_matches_torch_on_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_to_f64(codes.numpy())
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    assert nan.sum() == 2  # S.1111.111 only


def test_e4m3_anchor_codes_from_spec():
    for code, val in _read_table("e4m3_anchor_values.txt"):
        assert O.e4m3_to_f64(np.array([int(code, 16)]))[0] == val


def test_e4m3_encode_matches_torch_rne():
    g = torch.Generator().manual_seed(11)
    v = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-12, 8, (200000,), generator=g).float())
    v = v.clamp(-440, 440)
    # every midpoint between adjacent codes is a tie: RNE must pick the even code
    pos = torch.tensor(O.E4M3_TABLE[:127])
    mids = (pos[:-1] + pos[1:]) / 2
    v = torch.cat([v, mids.float(), -mids.float()])
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = O.f64_to_e4m3(v.double().numpy())
    # -0 and +0 both decode to zero; compare values, then codes away from zero
    assert np.array_equal(O.e4m3_to_f64(mine), O.e4m3_to_f64(ref))


def test_e4m3_saturates():
    v = np.array([448.0, 449.0, 464.0, 500.0, 1e6, -1e6])
    assert np.array_equal(O.e4m3_to_f64(O.f64_to_e4m3(v)), [448, 448, 448, 448, 448, -448])


def test_bf16_decode_all_codes_matches_torch():
    codes = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16)
    ref = codes.view(torch.bfloat16).to(torch.float64).numpy()
    mine = O.bf16_to_f64(codes.numpy())
    fin = np.isfinite(ref)
    assert np.array_equal(mine[fin], ref[fin])


def test_bf16_encode_matches_torch_rne():
    g = torch.Generator().manual_seed(12)
    v = torch.randn(300000, generator=g) * torch.exp2(torch.randint(-30, 30, (300000,), generator=g).float())
    # exact ties: a bf16 value plus half its spacing
    base = torch.randn(5000, generator=g).to(torch.bfloat16).float()
    half_ulp = torch.tensor(O.ulp_bf16(base.double().numpy()) / 2).float()
    v = torch.cat([v, base + half_ulp, base - half_ulp])
    ref = v.to(torch.bfloat16).view(torch.int16).numpy()
    mine = O.f64_to_bf16(v.double().numpy())
    assert np.array_equal(mine, ref)


def test_e2m1_values_from_spec_table():
    table = _read_table("e2m1_values.txt")
    codes = np.array([int(c) for c, _ in table])
    vals = np.array([v for _, v in table])
    assert np.array_equal(O.e2m1_to_f64(codes), vals)


def test_every_e2m1_value_is_exact_in_e4m3():
    """FP4 -> FP8 dequantisation is lossless ("解读 DeepSeek V4", FP4 QAT section)."""
    vals = O.e2m1_to_f64(np.arange(16))
    t = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(t, vals)
    assert np.array_equal(O.e4m3_to_f64(O.f64_to_e4m3(vals)), vals)


def test_e8m0_matches_torch():
    codes = torch.arange(255, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(O.e8m0_to_f64(codes.numpy()), ref)
    assert np.isnan(O.e8m0_to_f64(np.array([255]))[0])


def test_mxfp4_roundtrip_bound_and_exact_values():
    """Generator encoder + oracle decoder: each element lands on the nearest E2M1 value
    times the block scale 2^(floor(log2 amax) - 2); representable inputs come back exactly."""
    g = torch.Generator().manual_seed(13)
    v = torch.randn(64, 4 * 32, generator=g)
    codes, scales = wl.mxfp4_encode(v)
    deq = O.mxfp4_to_f64(codes.numpy(), scales.numpy())
    vb = v.double().numpy().reshape(64, 4, 32)
    amax = np.abs(vb).max(-1)
    X = np.floor(np.log2(amax)) - 2
    assert np.array_equal(scales.numpy().astype(np.int64) - 127, X.astype(np.int64))
    grid = O.e2m1_to_f64(np.arange(8))
    scaled = vb / np.exp2(X)[..., None]
    nearest = grid[np.abs(np.abs(scaled)[..., None] - grid).argmin(-1)] * np.sign(scaled)
    err = np.abs(deq.reshape(64, 4, 32) - nearest * np.exp2(X)[..., None])
    # ties may go either way between the two nearest values; otherwise exact
    tie = np.isclose(np.sort(np.abs(np.abs(scaled)[..., None] - grid), -1)[..., 0],
                     np.sort(np.abs(np.abs(scaled)[..., None] - grid), -1)[..., 1])
    assert np.all((err == 0) | tie)
    # exact values: scale 2^-1 times every E2M1 value
    ex = torch.tensor(np.tile(np.concatenate([grid, -grid[1:], [0.0]]), 2) * 0.5, dtype=torch.float32)
    ex = ex[None, :32]
    ex[0, 0] = 3.0  # amax 3 -> X = 2^(1-2) = 0.5
    c2, s2 = wl.mxfp4_encode(ex)
    assert np.array_equal(O.mxfp4_to_f64(c2.numpy(), s2.numpy()), ex.double().numpy())


def test_mxfp4_saturation_and_zero_block():
    v = torch.zeros(1, 64)
    v[0, 32] = 6.0
    v[0, 33] = -5.9  # amax 6: X = 2^0, -5.9 rounds to -6
    codes, scales = wl.mxfp4_encode(v)
    assert scales.tolist() == [[127, 127]]
    d = O.mxfp4_to_f64(codes.numpy(), scales.numpy())
    assert d[0, 32] == 6.0 and d[0, 33] == -6.0 and np.all(d[0, :32] == 0)


def test_e2m1_values_match_ml_dtypes():
    """The 16 E2M1 codes against ml_dtypes' float4_e2m1fn (an independent decoder of the
    OCP MX v1.0 element type)."""
    ml_dtypes = pytest.importorskip("ml_dtypes")
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(O.e2m1_to_f64(np.arange(16)), ref)


def test_mxfp4_decode_matches_an_independent_dequantizer_on_every_byte_and_scale():
    """Nibble order, element values and block scaling of the oracle's MXFP4 decoder
    against OpenAI's triton_kernels MXFP4 upcast (pure torch; vendored by vllm): all 256
    byte codes (16 blocks of 32 elements) under every E8M0 scale code 1..252.  Scale code
    0 is left out because that upcast maps it to 0 rather than 2^-127; codes 253 and 254
    overflow its FP32 output (6 * 2^126 > FP32 max); code 255 is NaN in OCP MX."""
    mx = pytest.importorskip("vllm.third_party.triton_kernels.numerics_details.mxfp")
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).reshape(16, 16)
    for s0 in range(1, 253, 16):
        sc = torch.clamp(torch.arange(s0, s0 + 16), max=252).to(torch.uint8).reshape(16, 1)
        ref = mx.upcast_from_mxfp_torch(codes, sc, torch.float32, axis=-1).double().numpy()
        mine = O.mxfp4_to_f64(codes.numpy(), sc.numpy())
        assert np.array_equal(mine, ref), f"scales {s0}..{s0 + 15}"
    # element 2i in the low nibble: byte 0x61 holds 0.5 (code 1) then 4.0 (code 6)
    assert np.array_equal(O.mxfp4_to_f64(np.full((1, 16), 0x61, np.uint8), np.array([[127]]))[0, :2], [0.5, 4.0])


def test_e2m1_encoder_matches_ml_dtypes_rounding():
    """The oracle's E2M1 conversion (nearest value, ties to the even code, saturating at
    +-6) against ml_dtypes' float4_e2m1fn cast, on random values and on every tie."""
    ml_dtypes = pytest.importorskip("ml_dtypes")
    rng = np.random.default_rng(21)
    grid = O.e2m1_to_f64(np.arange(8))
    ties = (grid[:-1] + grid[1:]) / 2
    v = np.concatenate([rng.standard_normal(20000) * 3, ties, -ties, [0.0, 6.0, 7.99, -7.99, 1e-9]])
    ref = v.astype(np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    mine = O.e2m1_to_f64(O.f64_to_e2m1(v))
    assert np.array_equal(mine, ref)
    assert np.all(O.f64_to_e2m1(np.array([-0.1, -0.0, 0.0])) == 0)  # zero is code 0


def test_mxfp4_encoder_scale_rule_and_elements():
    """OCP MX v1.0 shared scale X = 2^(floor(log2 amax) - 2) on crafted blocks, a zero block
    at 2^0, and elements equal to the E2M1 cast of v / X."""
    ml_dtypes = pytest.importorskip("ml_dtypes")
    blocks = np.zeros((5, 32))
    blocks[0, 3] = 1.0          # floor(log2 1) = 0 -> X = 2^-2
    blocks[1, 0] = -6.0         # 2 -> X = 2^0
    blocks[2, 31] = 0.3         # -2 -> X = 2^-4
    blocks[3, 7] = 1000.0       # 9 -> X = 2^7
    codes, scales = O.f64_to_mxfp4(blocks.reshape(1, 160))
    assert scales.tolist() == [[125, 127, 123, 134, 127]]
    rng = np.random.default_rng(22)
    v = rng.standard_normal((50, 128)) * np.exp2(rng.integers(-6, 6, (50, 1)))
    codes, scales = O.f64_to_mxfp4(v)
    X = np.exp2(scales.astype(np.float64) - 127)
    ref = (v.reshape(50, 4, 32) / X[..., None]).astype(np.float32).astype(ml_dtypes.float4_e2m1fn)
    assert np.array_equal(O.mxfp4_to_f64(codes, scales), ref.astype(np.float64).reshape(50, 128) * np.repeat(X, 32, -1))


def test_mxfp4_encoder_agrees_with_the_input_generator():
    """Two independent codings of the same rule: the oracle's (numpy distances) and the
    input generator's (torch bucketize), bit for bit on N(0,1) data."""
    g = torch.Generator().manual_seed(23)
    v = torch.randn(300, 128, generator=g)
    c1, s1 = wl.mxfp4_encode(v)
    c2, s2 = O.f64_to_mxfp4(v.double().numpy())
    assert np.array_equal(c1.numpy(), c2) and np.array_equal(s1.numpy(), s2)


def test_mxfp4_encoder_roundtrips_representable_values():
    grid = O.e2m1_to_f64(np.arange(16))
    rng = np.random.default_rng(24)
    v = rng.choice(grid, (20, 64)) * 0.125
    v[:, 0] = 6 * 0.125          # pin each block's amax so X = 2^-3
    v[:, 32] = -6 * 0.125
    c, s = O.f64_to_mxfp4(v)
    assert np.array_equal(O.mxfp4_to_f64(c, s), v)
