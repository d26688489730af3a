"""Grouped output projection (lc_grouped_out_proj, tcgen05 BF16 GEMM per group) against the
oracle, through the C ABI: each output within the FP32 accumulation bound of the float64
result plus the rounding of the output format."""
import numpy as np
import pytest
import torch

import long_context_sparse_softmax_b200 as lc
from oracle import lc_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_q,H,Dv,G,d_g,f32", [
    (300, 64, 512, 8, 512, False),    # values without RoPE dims, 8 groups -> 4096 outputs
    (32, 64, 576, 8, 96, True),       # a decode batch; d_g not a multiple of the 128-column tile
    (1000, 128, 512, 16, 256, False),
])
def test_grouped_projection_matches_oracle(n_q, H, Dv, G, d_g, f32):
    g = torch.Generator(device="cuda").manual_seed(n_q + G)
    K = (H // G) * Dv
    x = torch.randn(n_q, H, Dv, device="cuda", generator=g).to(torch.bfloat16)
    wt = (torch.randn(G, d_g, K, device="cuda", generator=g) / K ** 0.5).to(torch.bfloat16)  # W_g transposed
    y = torch.empty(n_q, G * d_g, device="cuda", dtype=torch.float32 if f32 else torch.bfloat16)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    a = lc.OutProjArgs(n_q, H, Dv, G, d_g, lc.LC_FMT_F32 if f32 else lc.LC_FMT_BF16, x.data_ptr(), wt.data_ptr(),
                       y.data_ptr(), status.data_ptr())
    lc.lc_grouped_out_proj(a)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    xd = x.double().cpu().numpy()
    wd = wt.double().cpu().numpy().transpose(0, 2, 1)             # [G, K, d_g]
    ref = O.grouped_out_proj(xd, wd)
    mag = O.grouped_out_proj(np.abs(xd), np.abs(wd))              # sum of |terms|
    bound = K * 2.0 ** -24 * mag + (0 if f32 else O.ulp_bf16(np.abs(ref)))
    got = y.double().cpu().numpy()
    err = np.abs(got - ref)
    assert np.all(err <= bound + 1e-12), f"max err / bound {np.max(err / (bound + 1e-30))}"
