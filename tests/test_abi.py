"""C-ABI checks that need no GPU: the library loads, exports every entry point that
include/lc.h declares, its struct layouts match the binding, and host-side validation
rejects bad arguments before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

import long_context_sparse_softmax_b200 as lc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lc.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[a-z_ ]+\*?\s*\b(lc_[a-z0-9_]+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for op in ("qk_prep", "csa_compress", "hca_compress", "csa_index_scores", "csa_topk",
               "csa_sparse_attn", "hca_attn"):
        assert f"lc_{op}_prefill" in names and f"lc_{op}_decode" in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", lc.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT (lc_[a-z0-9_]+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(lc.lib, n)


def test_struct_layouts_match_binding():
    for i, st in enumerate(lc.STRUCTS):
        assert lc.lib.lc_struct_size(i) == ctypes.sizeof(st)
    assert lc.lib.lc_struct_size(99) == 0


def test_version_and_status_strings():
    assert "sm_100a" in lc.lc_version()
    for s in range(7):
        assert lc.lib.lc_status_string(s).decode().startswith("LC_")


def _raw(name, args):
    return getattr(lc.lib, name)(ctypes.byref(args) if args is not None else None, None)


def test_null_args_rejected():
    for name in lc.ENTRY_POINTS:
        assert getattr(lc.lib, name)(None, None) == lc.LC_ERR_ARG


def test_bad_dims_rejected_without_launch():
    a = lc.QkPrepArgs()
    a.dims = lc.Dims(100, 64, 0, 1)  # D not a multiple of 8
    a.n_tok, a.in_fmt = 4, lc.LC_FMT_BF16
    assert _raw("lc_qk_prep_prefill", a) == lc.LC_ERR_ARG
    a.dims = lc.Dims(576, 64, 520, 1)  # RoPE range past D
    assert _raw("lc_qk_prep_prefill", a) == lc.LC_ERR_ARG
    a.dims = lc.Dims(576, 64, 512, 1)
    a.out = lc.Rows(lc.LC_FMT_E4M3_BF16, 0, 16, None)  # split format without its RoPE part
    a.x, a.pos = 16, 16
    assert _raw("lc_qk_prep_prefill", a) == lc.LC_ERR_ARG
    a.out = lc.Rows(lc.LC_FMT_BF16, 0, 24, None)  # misaligned
    assert _raw("lc_qk_prep_prefill", a) == lc.LC_ERR_ALIGN


def test_compress_ratio_ranges():
    a = lc.CompressArgs()
    a.dims = lc.Dims(576, 64, 512, 1)
    a.in_fmt = lc.LC_FMT_BF16
    a.m = 128
    assert _raw("lc_csa_compress_prefill", a) == lc.LC_ERR_ARG  # CSA takes m <= 64
    a.m = 4
    assert _raw("lc_hca_compress_prefill", a) == lc.LC_ERR_ARG  # HCA takes m >= 64
    a.m, a.num_seqs, a.max_blocks = 128, 0, 0
    assert _raw("lc_hca_compress_prefill", a) == lc.LC_OK        # nothing to do, no launch


def test_index_format_checks():
    a = lc.IndexArgs()
    a.n_q, a.H_I, a.d_I, a.fmt, a.m, a.max_ent, a.score_stride = 1, 64, 96, lc.LC_IDX_MXFP4, 4, 8, 8
    assert _raw("lc_csa_index_scores_prefill", a) == lc.LC_ERR_UNSUPPORTED
    a.d_I, a.score_stride = 128, 6
    assert _raw("lc_csa_index_scores_prefill", a) == lc.LC_ERR_ARG  # stride < max_ent
    a.score_stride = 8
    a.batch.num_seqs = 2
    assert _raw("lc_csa_index_scores_decode", a) == lc.LC_ERR_ARG  # decode: one query per sequence
    a.fmt = 7
    assert _raw("lc_csa_index_scores_prefill", a) == lc.LC_ERR_ARG


def test_topk_and_attention_checks():
    t = lc.TopkArgs()
    t.n_q, t.k, t.m, t.max_ent, t.score_stride = 1, 0, 4, 8, 8
    assert _raw("lc_csa_topk_prefill", t) == lc.LC_ERR_ARG   # k >= 1
    a = lc.AttnArgs()
    a.dims = lc.Dims(576, 64, 512, 64)
    a.n_q, a.k, a.m, a.W, a.max_ent, a.out_fmt = 1, 0, 4, 128, 8, lc.LC_FMT_BF16
    assert _raw("lc_csa_sparse_attn_prefill", a) == lc.LC_ERR_ARG  # CSA needs k >= 1
    a.k, a.out_fmt = 8, lc.LC_FMT_E4M3_BF16
    assert _raw("lc_csa_sparse_attn_prefill", a) == lc.LC_ERR_ARG  # output is F32 or BF16


def test_binding_raises_on_error_status():
    with pytest.raises(lc.LcError) as e:
        lc.lc_csa_topk_prefill(lc.TopkArgs(), 0)
    assert e.value.status == lc.LC_ERR_ARG
    with pytest.raises(TypeError):
        lc.lc_csa_topk_prefill(lc.AttnArgs(), 0)


def test_attention_workspace_sizes_on_the_host():
    """The size queries read only host fields.  HCA prefill with BF16 queries (the
    F16-operand kernel) offers an F16 image of the entries, 73,728 bytes per 64 entry
    rows; nothing where that kernel does not run or the entry rows are unknown."""
    a = lc.AttnArgs()
    a.dims = lc.Dims(576, 64, 512, 64)
    a.n_q, a.m, a.W, a.max_ent, a.out_fmt = 4096, 128, 128, 8192, lc.LC_FMT_BF16
    a.q = lc.Rows(fmt=lc.LC_FMT_BF16)
    a.ent = lc.Rows(fmt=lc.LC_FMT_E4M3_BF16)
    a.win = lc.Rows(fmt=lc.LC_FMT_BF16)
    size = lc.lc_hca_attn_prefill_workspace_bytes
    a.n_ent_rows = 8192
    assert size(a) == 128 * 73728
    a.n_ent_rows = 8193
    assert size(a) == 129 * 73728
    a.n_ent_rows = 0
    assert size(a) == 0
    a.n_ent_rows = 8192
    assert lc.lc_hca_attn_workspace_bytes(a) == 0  # decode sizes: 4096 queries split no keys
    a.impl = lc.LC_IMPL_REF
    assert size(a) == 0
    a.impl = lc.LC_IMPL_AUTO
    a.q = lc.Rows(fmt=lc.LC_FMT_E4M3_BF16)  # E4M3 queries: the E4M3-score kernel
    a.n_win_rows = 128
    assert size(a) == 0
