"""Host-side pieces of the bench and the runner that need no GPU: the tensor peaks per
stage, the config both bench arms report, and which per-step inputs each stage reads."""
import pytest

import bench
from long_context_sparse_softmax_b200 import runner
from long_context_sparse_softmax_b200 import workloads as wl


def test_tensor_peak_factors_follow_the_operand_types():
    csa_p, hca_p = wl.WORKLOADS["csa_prefill"][0], wl.WORKLOADS["hca_prefill"][0]
    # the MXFP4 indexer runs at 4x the BF16 rate
    assert bench.tensor_mix("0:index", csa_p)[0] == 4.0
    # E4M3 scores + F16 P V: half the flops at 2x, half at 1x
    assert bench.tensor_mix("0:attn", csa_p)[0] == pytest.approx(4.0 / 3.0)
    assert bench.tensor_mix("0:attn", hca_p)[0] == 1.0          # BF16 queries: the F16 kernel
    # a tensor-bound stage's roofline time uses that factor
    work = {"0:index": (1.0, 4.0e12)}
    pk = {"hbm_gbs": 1e9, "bf16_tflops": 1000.0}
    bnd, t = bench.bound_of("0:index", csa_p, work, pk)
    assert bnd == "tensor" and t == pytest.approx(4.0e12 / (4000.0e12))


def test_both_arms_report_one_config():
    c = bench.workload_config("csa_decode")
    assert c == {"workload": "csa_decode_b32_L131072_k512", "batch": 32, "context": 131072, "heads": 64,
                 "dims": 576, "topk": 512, "query_tokens_per_step_per_gpu": 32}
    assert bench.workload_config("mixed_decode")["workload"] == "mixed_decode"


def test_host_inputs_name_the_stage_that_reads_them():
    s = wl.shrink(wl.CSA_DECODE, name="host_io_decode", seq_lens=(512, 700), k=64)
    inp = wl.make_decode(s, "cpu")
    r = runner.Decode(inp, "cpu")
    h = r.host_inputs()
    assert h["qk_prep_q"][0] is inp["q_raw"]
    assert h["qk_prep_win"][0] is inp["x_new"]
    assert h["compress"][0] is inp["x_tail"] and h["compress"][1] is inp["g_tail"]
    # MXFP4 indexer: the step quantises the raw query rows and pools + quantises the key
    # of the closed block; index and top-k run fused
    assert r.fused and [n for n, _ in r.stages()][3:] == ["index_compress", "quant_q", "index_topk", "attn"]
    assert h["quant_q"][0] is inp["qI_raw"] and h["index_compress"][0] is inp["kI_tail"]
    side, main, after = r.dag()
    assert [[n for n, _ in g] for g in side] == [["qk_prep_q"], ["qk_prep_win"], ["compress", "index_compress"]]
    assert [n for n, _ in main] == ["quant_q", "index_topk"] and after[0][0] == "attn"
    r2 = runner.Decode(inp, "cpu", fused=False)
    assert [n for n, _ in r2.stages()][3:] == ["index_compress", "quant_q", "index", "topk", "attn"]
    assert r.host_outputs() == [r.out, r.lse]
    # prefill: the raw tokens feed both window preparation and compression (two side
    # streams), so they are copied before the fork
    p = wl.shrink(wl.CSA_PREFILL, name="host_io_prefill", seq_lens=(600,), H=16, k=32, n_q=600)
    ip = wl.make_prefill(p, "cpu")
    rp = runner.Prefill(ip, "cpu")
    hp = rp.host_inputs()
    assert hp["_fork"][0] is ip["x"] and hp["_fork"][1] is ip["g"]
    assert "qk_prep_win" not in hp and "compress" not in hp
    # prefill compresses the indexer keys on the main stream, before the indexer reads them
    assert hp["index_compress"][0] is ip["kI_raw"] and hp["quant_q"][0] is ip["qI_raw"]
    assert [n for n, _ in rp.dag()[1]] == ["index_compress", "quant_q", "index_topk"]


def test_runner_keeps_fused_topk_only_for_small_merges():
    """The fused index + top-k call is the default while its merge takes at most
    FUSED_MAX_CANDIDATES candidates per query (n_chunks x k, read from the call's
    workspace size); a long two-sequence batch with k = 1024 spreads each query over many
    key ranges and gets the separate calls; an explicit fused=True is kept."""
    long_ = wl.shrink(wl.MIXED_CSA, name="fused_choice_long", seq_lens=(200000, 160000), k=1024)
    inp = wl.make_decode(long_, "cpu")
    r = runner.Decode(inp, "cpu")
    assert not r.fused and [n for n, _ in r.stages()][-3:] == ["index", "topk", "attn"]
    assert runner.Decode(inp, "cpu", fused=True).fused
    short = wl.shrink(wl.CSA_DECODE, name="fused_choice_short", seq_lens=(4096, 3000), k=512)
    assert runner.Decode(wl.make_decode(short, "cpu"), "cpu").fused


@pytest.mark.parametrize("name", ["csa_decode", "csa_prefill", "hca_prefill", "mixed_decode", "tiny_csa_prefill"])
@pytest.mark.parametrize("fused", [None, False])
def test_stage_work_covers_every_stage(name, fused):
    """The bench counts algorithmic bytes / flops for every stage a step runs."""
    import dataclasses
    for spec in wl.WORKLOADS[name]:
        small = dataclasses.replace(spec, name="sw", seq_lens=tuple(min(L, 3000) for L in spec.seq_lens),
                                    **({} if spec.is_decode else {"n_q": 64, "q_first": min(spec.seq_lens[0], 3000) - 64}))
        inp = (wl.make_decode if small.is_decode else wl.make_prefill)(small, "cpu")
        r = (runner.Decode if small.is_decode else runner.Prefill)(inp, "cpu", fused=fused)
        work, units = bench.stage_work(small, inp, r)
        names = [n for n, _ in r.stages()]
        assert all(n in work for n in names), [n for n in names if n not in work]
        assert units == (small.num_seqs if small.is_decode else small.n_q)
