"""GPU parity at oracle-sized shapes: every query of each case is checked, the shapes
span several kernel tiles with ragged tails, and the edge cases of the method are
covered (no visible entry, fewer visible entries than k, window off, overlap reading,
sequences shorter than the window, m = 1)."""
import pytest

from long_context_sparse_softmax_b200 import workloads as wl
from tests.gpu_checks import check_decode, check_prefill

pytestmark = pytest.mark.gpu


def test_tiny_fp32_csa_prefill_all_queries():
    """The FP32 workload (L = 1024, D = 128, 8 heads, k = 64): top-k bit-exact,
    attention within 1e-4."""
    rep = check_prefill(wl.TINY_CSA_PREFILL)
    assert rep["topk_e2e_set_diff"] == 0


SMALL_CSA = wl.shrink(wl.CSA_PREFILL, name="small_csa_prefill", seed=31, seq_lens=(1100,), H=16, k=64,
                      n_q=1100, q_first=0)


def test_small_csa_prefill_fp8_mxfp4():
    check_prefill(SMALL_CSA)


def test_small_csa_prefill_128_heads_ragged():
    s = wl.shrink(wl.CSA_PREFILL, name="small_csa_h128", seed=32, seq_lens=(613,), H=128, k=32, n_q=613)
    check_prefill(s)


def test_small_csa_prefill_overlap_reading():
    check_prefill(SMALL_CSA, q_sel=range(0, 1100, 7), W_x=0)


def test_small_csa_prefill_without_window():
    s = wl.shrink(SMALL_CSA, name="small_csa_w0", seed=33, W=0, seq_lens=(300,), n_q=300)
    check_prefill(s)


def test_m1_fp32_csa_prefill():
    s = wl.shrink(wl.TINY_CSA_PREFILL, name="tiny_m1", seed=34, m=1, seq_lens=(300,), n_q=300, k=300)
    check_prefill(s)


def test_small_hca_prefill():
    s = wl.shrink(wl.HCA_PREFILL, name="small_hca_prefill", seed=35, seq_lens=(128 * 30 + 77,),
                  q_first=128 * 30 + 77 - 300, n_q=300)
    check_prefill(s)


def test_small_hca_prefill_from_position_zero():
    s = wl.shrink(wl.HCA_PREFILL, name="small_hca_from0", seed=36, seq_lens=(700,), q_first=0, n_q=700)
    check_prefill(s)


def test_small_csa_decode_ragged():
    s = wl.shrink(wl.CSA_DECODE, name="small_csa_decode", seed=37, seq_lens=(1000, 2053, 517, 50, 132), k=128)
    check_decode(s)


def test_small_csa_decode_k1024():
    s = wl.shrink(wl.MIXED_CSA, name="small_mixed_csa", seed=38, seq_lens=(5000, 4096, 1300))
    check_decode(s)


def test_small_hca_decode_ragged():
    s = wl.shrink(wl.MIXED_HCA, name="small_hca_decode", seed=39, seq_lens=(128 * 20 + 5, 128 * 3, 1000, 64))
    check_decode(s)


def test_small_csa_decode_overlap_reading():
    s = wl.shrink(wl.CSA_DECODE, name="small_csa_decode_ov", seed=40, seq_lens=(900, 1204), k=64)
    check_decode(s, W_x=0)


# every attention kernel on the same shapes (the tests above use the automatic choice)
IMPLS = [pytest.param(2, id="tcgen05"), pytest.param(3, id="reference")]


@pytest.mark.parametrize("impl", IMPLS)
def test_small_csa_prefill_each_attention_kernel(impl):
    s = wl.shrink(wl.CSA_PREFILL, name="small_csa_impl", seed=41, seq_lens=(700,), H=64, k=96, n_q=700)
    check_prefill(s, q_sel=range(0, 700, 3), impl=impl)


@pytest.mark.parametrize("impl", IMPLS)
def test_small_hca_prefill_each_attention_kernel(impl):
    s = wl.shrink(wl.HCA_PREFILL, name="small_hca_impl", seed=42, seq_lens=(128 * 24 + 50,),
                  q_first=128 * 24 + 50 - 160, n_q=160)
    check_prefill(s, impl=impl)


@pytest.mark.parametrize("impl", IMPLS)
def test_small_csa_decode_each_attention_kernel(impl):
    s = wl.shrink(wl.CSA_DECODE, name="small_decode_impl", seed=43, seq_lens=(3000, 1027, 8192, 200), k=256)
    check_decode(s, impl=impl)


@pytest.mark.parametrize("impl", IMPLS)
def test_small_hca_decode_each_attention_kernel(impl):
    s = wl.shrink(wl.MIXED_HCA, name="small_hcad_impl", seed=44, seq_lens=(128 * 40 + 3, 900, 128 * 7))
    check_decode(s, impl=impl)


def test_per_query_indexer_weights_decode_and_prefill():
    """Indexer head weights given per query ([n_q, H_I], w_qstride = H_I) instead of shared."""
    check_decode(wl.shrink(wl.CSA_DECODE, name="wq_decode", seed=45, seq_lens=(3000, 1027, 9000), k=128,
                           w_per_query=True))
    check_prefill(wl.shrink(wl.CSA_PREFILL, name="wq_prefill", seed=46, seq_lens=(900,), H=64, k=64, n_q=900,
                            w_per_query=True), q_sel=range(0, 900, 5))


# values without the RoPE dims (outputs of D - d_r dims), on every attention kernel
@pytest.mark.parametrize("impl", IMPLS)
def test_nope_values_csa_decode(impl):
    s = wl.shrink(wl.CSA_DECODE, name="vnope_decode", seed=47, seq_lens=(3000, 1027, 8192, 200), k=256, v_nope=True)
    check_decode(s, impl=impl)


def test_nope_values_csa_decode_few_queries_combine():
    """Two queries: more key splits than a cluster holds, so the partials are merged by the
    combine kernel."""
    check_decode(wl.shrink(wl.CSA_DECODE, name="vnope_combine", seed=48, seq_lens=(20000, 9001), k=512,
                           v_nope=True))


def test_nope_values_prefill_kernels():
    check_prefill(wl.shrink(wl.CSA_PREFILL, name="vnope_csa_prefill", seed=49, seq_lens=(700,), H=64, k=96, n_q=700,
                            v_nope=True), q_sel=range(0, 700, 3))
    check_prefill(wl.shrink(wl.HCA_PREFILL, name="vnope_hca_prefill", seed=50, seq_lens=(128 * 24 + 50,),
                            q_first=128 * 24 + 50 - 160, n_q=160, v_nope=True))
    check_prefill(wl.shrink(wl.TINY_CSA_PREFILL, name="vnope_tiny", seed=51, seq_lens=(400,), n_q=400, v_nope=True))


def test_csa_decode_f32_output_cluster_merge():
    """FP32 outputs of the decode path whose key splits merge over a thread-block cluster
    (few queries, so each query's keys are split over several CTAs).  The FP32 result must
    round to the BF16 run's result within one BF16 step (the BF16 run is checked against
    the oracle by the tests above) and be finite."""
    import numpy as np
    import torch
    from long_context_sparse_softmax_b200 import runner
    base = wl.shrink(wl.CSA_DECODE, name="f32_out_cluster", seed=42, seq_lens=(3000, 5200, 2100), k=128)
    inp = wl.make_decode(base, "cuda")
    r16 = runner.Decode(inp, "cuda")
    r16.step()
    inp32 = dict(inp)
    inp32["spec"] = wl.shrink(base, out32=True)
    r32 = runner.Decode(inp32, "cuda")
    r32.step()
    torch.cuda.synchronize()
    assert r16.read_status() == 0 and r32.read_status() == 0
    o16 = (r16.out.to(torch.int32) << 16).view(torch.float32).cpu().numpy().astype(np.float64)
    o32 = r32.out.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o32))
    rms = np.sqrt(np.mean(o32 * o32, axis=-1, keepdims=True))
    # BF16 rounding (at most 2^-9 relative, round to nearest) of the same FP32 sum; the
    # margin covers a different summation order
    assert np.all(np.abs(o16 - o32) <= 2.0 ** -8 * np.abs(o32) + 2.0 ** -12 * rms + 1e-30)


def test_hca_prefill_entry_image_is_bit_identical():
    """With its optional workspace, dense prefill widens the entries to F16 once and reads
    each 64 visible entries as one tile of that image; without it, every query gathers and
    widens its own tiles.  Both give the same bits.  Here 200 entries give three image
    tiles, then a gathered tile of the last visible entries and the window."""
    import torch
    from long_context_sparse_softmax_b200 import runner
    L = 128 * 200 + 77
    s = wl.shrink(wl.HCA_PREFILL, name="hca_image", seed=52, seq_lens=(L,), q_first=L - 96, n_q=96)
    check_prefill(s, q_sel=range(0, 96, 5))
    run = runner.Prefill(wl.make_prefill(s, "cuda"), "cuda")
    n_rows = run.a_attn.n_ent_rows
    assert n_rows >= 200 and run.a_attn.workspace_bytes == (n_rows + 63) // 64 * 64 * 1152
    run.step()
    torch.cuda.synchronize()
    assert run.read_status() == 0
    out_img, lse_img = run.out.clone(), run.lse.clone()
    run.a_attn.workspace_bytes = 0  # the per-query gather path
    run.attn()
    torch.cuda.synchronize()
    assert run.read_status() == 0
    assert torch.equal(out_img, run.out) and torch.equal(lse_img, run.lse)
