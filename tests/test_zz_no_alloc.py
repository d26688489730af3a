"""The allocation-free decode attention entry point (lc_csa_sparse_attn_decode_static).

Some callers cannot allocate device memory when they call the library: hosts that give
all device memory to their own allocator up front, and latency-bound serving loops that
must not pay for cudaMalloc's synchronisation.  For them the library keeps the decode
attention's scratch in a fixed array compiled into it.  This test checks, through the C
ABI, that two calls in a row of that entry point give the same attention as the regular
entry point that takes a caller-allocated workspace.  It builds its own inputs, so it
runs alone or after the other tests; this file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import long_context_sparse_softmax_b200 as lc
from long_context_sparse_softmax_b200 import runner
from long_context_sparse_softmax_b200 import workloads as wl
from tests.oracle_ref import attn_ok, np_
from oracle import lc_oracle as O

pytestmark = pytest.mark.gpu

# ragged batch whose decode attention splits keys across CTAs, so the scratch is used
SPEC = wl.shrink(wl.CSA_DECODE, name="static_scratch_decode", seed=71, seq_lens=(20000, 9001, 131072, 4099))


def _bf16(t: torch.Tensor) -> np.ndarray:
    return O.bf16_to_f64(np_(t))


def test_static_scratch_matches_workspace_entry_on_two_calls():
    inp = wl.make_decode(SPEC, "cuda")
    run = runner.Decode(inp, "cuda")
    run.step()
    torch.cuda.synchronize()
    assert run.read_status() == 0
    need = lc.lc_csa_sparse_attn_workspace_bytes(run.a_attn)
    assert 0 < need <= lc.lc_csa_sparse_attn_decode_static_capacity()
    ref_out = _bf16(run.out).reshape(SPEC.num_seqs, SPEC.H, SPEC.D)
    ref_lse = np_(run.lse).reshape(SPEC.num_seqs, SPEC.H)
    for call in range(2):
        out = torch.full_like(run.out, 0x7fc0)   # BF16 NaN: every element must be written
        lse = torch.full_like(run.lse, float("nan"))
        a = lc.AttnArgs.from_buffer_copy(run.a_attn)
        a.out, a.lse = out.data_ptr(), lse.data_ptr()
        a.workspace, a.workspace_bytes = None, 0
        lc.lc_csa_sparse_attn_decode_static(a)
        torch.cuda.synchronize()
        assert run.read_status() == 0
        got = _bf16(out).reshape(SPEC.num_seqs, SPEC.H, SPEC.D)
        got_lse = np_(lse).reshape(SPEC.num_seqs, SPEC.H)
        assert np.all(np.isfinite(got)) and np.all(np.isfinite(got_lse)), f"call {call}: output not written"
        for b in range(SPEC.num_seqs):
            ok, err, tol = attn_ok(got[b], ref_out[b], False)
            assert ok, f"call {call}, sequence {b}: err {err} > tol {tol}"
        np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=2e-3)


def test_static_scratch_rejects_requests_beyond_its_capacity():
    # 64 queries x 64 heads with top-k 8192: two key splits need ~18.9 MB > 16 MiB
    a = lc.AttnArgs()
    a.dims = lc.Dims(576, 64, 512, 64)
    a.n_q, a.k, a.m, a.W, a.W_x, a.max_ent = 64, 8192, 4, 128, 128, 1 << 18
    a.scale, a.out_fmt = 1 / 24, lc.LC_FMT_BF16
    a.q = a.ent = lc.Rows(lc.LC_FMT_E4M3_BF16, 0, 16, 16)
    a.win = lc.Rows(lc.LC_FMT_BF16, 0, 16, None)
    a.batch.num_seqs = 64
    assert lc.lc_csa_sparse_attn_workspace_bytes(a) > lc.lc_csa_sparse_attn_decode_static_capacity()
    with pytest.raises(lc.LcError) as e:
        lc.lc_csa_sparse_attn_decode_static(a, 0)
    assert e.value.status == lc.LC_ERR_TOO_LARGE
