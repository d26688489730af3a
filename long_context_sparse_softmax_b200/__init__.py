"""CSA / HCA long-context sparse attention for NVIDIA B200 — Python binding of liblc.so.

The binding only marshals arguments: every step of the path runs in the library's CUDA
kernels.  There is no CPU fallback.  liblc.so is loaded on first use (the first call, or
the first access to ``lib``), and that use raises ImportError if the library is missing
(build it with ``python long_context_sparse_softmax_b200/build_lib.py``).  Importing the
package alone loads nothing, so its input generators (``workloads``) can be used by a
process that never touches the GPU library.

Each C entry point ``lc_<op>_<variant>(const args*, stream)`` is exposed under the same
name; it takes the ctypes mirror of the args struct and an optional torch stream and
raises LcError on a non-zero status.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_float, c_int32, c_int64, c_size_t, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblc.so")

LC_OK, LC_ERR_ARG, LC_ERR_ALIGN, LC_ERR_UNSUPPORTED, LC_ERR_WORKSPACE, LC_ERR_LAUNCH, LC_ERR_TOO_LARGE = range(7)
LC_DEV_BAD_INDEX, LC_DEV_WINDOW_RANGE, LC_DEV_BAD_BLOCK, LC_DEV_NONVISIBLE, LC_DEV_TIMEOUT, LC_DEV_RANGE = \
    1, 2, 4, 8, 16, 32
LC_FMT_F32, LC_FMT_BF16, LC_FMT_E4M3_BF16 = 0, 1, 2
LC_IDX_F32, LC_IDX_MXFP4, LC_IDX_MXFP4_QBF16 = 0, 3, 4


class LcError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {load().lc_status_string(status).decode()} (status {status})")
        self.status = status


class Rows(ctypes.Structure):
    _fields_ = [("fmt", c_int32), ("reserved", c_int32), ("x", c_void_p), ("rope", c_void_p)]


class Dims(ctypes.Structure):
    _fields_ = [("D", c_int32), ("d_r", c_int32), ("rope_off", c_int32), ("H", c_int32)]


class Batch(ctypes.Structure):
    _fields_ = [("num_seqs", c_int32), ("win_ring", c_int32), ("q_start", c_void_p), ("q_pos0", c_void_p),
                ("ent_start", c_void_p), ("n_ent", c_void_p), ("win_start", c_void_p), ("win_pos0", c_void_p),
                ("win_len", c_void_p)]


class QkPrepArgs(ctypes.Structure):
    _fields_ = [("dims", Dims), ("n_tok", c_int32), ("in_fmt", c_int32), ("x", c_void_p), ("pos", c_void_p),
                ("out_tok", c_void_p), ("out", Rows), ("eps", c_float), ("rope_base", c_float),
                ("status", c_void_p)]


class CompressArgs(ctypes.Structure):
    _fields_ = [("dims", Dims), ("m", c_int32), ("num_seqs", c_int32), ("in_fmt", c_int32), ("max_blocks", c_int32),
                ("x", c_void_p), ("g", c_void_p), ("tok_row0", c_void_p), ("tok_pos0", c_void_p),
                ("tok_len", c_void_p), ("blk_first", c_void_p), ("blk_count", c_void_p), ("ent_start", c_void_p),
                ("out", Rows), ("eps", c_float), ("rope_base", c_float), ("status", c_void_p)]


class IndexArgs(ctypes.Structure):
    _fields_ = [("n_q", c_int32), ("H_I", c_int32), ("d_I", c_int32), ("fmt", c_int32), ("q", c_void_p),
                ("q_scale", c_void_p), ("k", c_void_p), ("k_scale", c_void_p), ("n_keys", c_int64), ("w", c_void_p),
                ("w_qstride", c_int32), ("m", c_int32), ("W_x", c_int32), ("max_ent", c_int32), ("batch", Batch),
                ("scores", c_void_p), ("score_stride", c_int64), ("status", c_void_p), ("spin_limit", c_int32),
                ("pdl", c_int32)]


class TopkArgs(ctypes.Structure):
    _fields_ = [("n_q", c_int32), ("k", c_int32), ("m", c_int32), ("W_x", c_int32), ("max_ent", c_int32),
                ("pdl", c_int32), ("scores", c_void_p), ("score_stride", c_int64), ("batch", Batch),
                ("idx", c_void_p), ("count", c_void_p), ("status", c_void_p)]


class IndexTopkArgs(ctypes.Structure):
    _fields_ = [("index", IndexArgs), ("k", c_int32), ("reserved", c_int32), ("idx", c_void_p), ("count", c_void_p),
                ("workspace", c_void_p), ("workspace_bytes", c_size_t)]


class Mxfp4QuantArgs(ctypes.Structure):
    _fields_ = [("n_rows", c_int64), ("d", c_int32), ("in_fmt", c_int32), ("x", c_void_p), ("codes", c_void_p),
                ("scales", c_void_p)]


class IndexCompressArgs(ctypes.Structure):
    _fields_ = [("d_I", c_int32), ("m", c_int32), ("num_seqs", c_int32), ("in_fmt", c_int32), ("max_blocks", c_int32),
                ("reserved", c_int32), ("x", c_void_p), ("g", c_void_p), ("tok_row0", c_void_p), ("tok_pos0", c_void_p),
                ("tok_len", c_void_p), ("blk_first", c_void_p), ("blk_count", c_void_p), ("ent_start", c_void_p),
                ("codes", c_void_p), ("scales", c_void_p), ("status", c_void_p)]


class OutProjArgs(ctypes.Structure):
    _fields_ = [("n_q", c_int32), ("H", c_int32), ("Dv", c_int32), ("G", c_int32), ("d_g", c_int32), ("out_fmt", c_int32),
                ("x", c_void_p), ("w", c_void_p), ("y", c_void_p), ("status", c_void_p)]


class AttnArgs(ctypes.Structure):
    _fields_ = [("dims", Dims), ("n_q", c_int32), ("k", c_int32), ("m", c_int32), ("W", c_int32), ("W_x", c_int32),
                ("max_ent", c_int32), ("scale", c_float), ("out_fmt", c_int32), ("q", Rows), ("ent", Rows),
                ("win", Rows), ("idx", c_void_p), ("sink", c_void_p), ("batch", Batch), ("out", c_void_p),
                ("lse", c_void_p), ("workspace", c_void_p), ("workspace_bytes", c_size_t), ("status", c_void_p),
                ("impl", c_int32), ("n_ent_rows", c_int32),
                ("n_win_rows", c_int32), ("v_nope", c_int32), ("pdl", c_int32)]


LC_IMPL_AUTO, LC_IMPL_TC, LC_IMPL_REF = 0, 2, 3


STRUCTS = [Rows, Dims, Batch, QkPrepArgs, CompressArgs, IndexArgs, TopkArgs, AttnArgs, IndexTopkArgs, Mxfp4QuantArgs,
           IndexCompressArgs, OutProjArgs]

ENTRY_POINTS = {
    "lc_qk_prep_prefill": QkPrepArgs, "lc_qk_prep_decode": QkPrepArgs,
    "lc_csa_compress_prefill": CompressArgs, "lc_csa_compress_decode": CompressArgs,
    "lc_hca_compress_prefill": CompressArgs, "lc_hca_compress_decode": CompressArgs,
    "lc_csa_index_scores_prefill": IndexArgs, "lc_csa_index_scores_decode": IndexArgs,
    "lc_csa_topk_prefill": TopkArgs, "lc_csa_topk_decode": TopkArgs,
    "lc_csa_index_topk_prefill": IndexTopkArgs, "lc_csa_index_topk_decode": IndexTopkArgs,
    "lc_mxfp4_quantize": Mxfp4QuantArgs,
    "lc_grouped_out_proj": OutProjArgs,
    "lc_csa_index_compress_prefill": IndexCompressArgs, "lc_csa_index_compress_decode": IndexCompressArgs,
    "lc_csa_sparse_attn_prefill": AttnArgs, "lc_csa_sparse_attn_decode": AttnArgs,
    "lc_hca_attn_prefill": AttnArgs, "lc_hca_attn_decode": AttnArgs,
    "lc_csa_sparse_attn_decode_static": AttnArgs,
}
HELPERS = ["lc_csa_sparse_attn_workspace_bytes", "lc_hca_attn_workspace_bytes", "lc_hca_attn_prefill_workspace_bytes",
           "lc_csa_index_topk_workspace_bytes",
           "lc_version",
           "lc_status_string", "lc_struct_size", "lc_csa_sparse_attn_decode_static_capacity"]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"liblc.so not built at {LIB_PATH}; run python long_context_sparse_softmax_b200/build_lib.py")
    so = ctypes.CDLL(LIB_PATH)
    for name, st in ENTRY_POINTS.items():
        fn = getattr(so, name)
        fn.argtypes = [ctypes.POINTER(st), c_void_p]
        fn.restype = c_int32
    for name in ("lc_csa_sparse_attn_workspace_bytes", "lc_hca_attn_workspace_bytes",
                 "lc_hca_attn_prefill_workspace_bytes"):
        fn = getattr(so, name)
        fn.argtypes = [ctypes.POINTER(AttnArgs)]
        fn.restype = c_size_t
    so.lc_csa_index_topk_workspace_bytes.argtypes = [ctypes.POINTER(IndexTopkArgs), c_int32]
    so.lc_csa_index_topk_workspace_bytes.restype = c_size_t
    so.lc_csa_sparse_attn_decode_static_capacity.restype = c_size_t
    so.lc_version.restype = ctypes.c_char_p
    so.lc_status_string.argtypes = [c_int32]
    so.lc_status_string.restype = ctypes.c_char_p
    so.lc_struct_size.argtypes = [c_int32]
    so.lc_struct_size.restype = c_size_t
    for i, st in enumerate(STRUCTS):
        if so.lc_struct_size(i) != ctypes.sizeof(st):
            raise ImportError(f"{st.__name__}: binding size {ctypes.sizeof(st)} != library {so.lc_struct_size(i)}")
    return so


_LIB = None


def load() -> ctypes.CDLL:
    """The loaded liblc.so (loaded and checked on the first call)."""
    global _LIB
    if _LIB is None:
        _LIB = _load()
    return _LIB


def __getattr__(name):
    if name == "lib":
        return load()
    raise AttributeError(name)


def _stream_handle(stream) -> c_void_p:
    if stream is None:
        import torch
        return c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return c_void_p(stream)
    return c_void_p(stream.cuda_stream)


def _make_call(name: str, st):
    def call(args, stream=None):
        if not isinstance(args, st):
            raise TypeError(f"{name} takes {st.__name__}")
        s = getattr(load(), name)(ctypes.byref(args), _stream_handle(stream))
        if s != LC_OK:
            raise LcError(s, name)

    call.__name__ = name
    call.__doc__ = f"{name}(args: {st.__name__}, stream=None): see include/lc.h"
    return call


for _n, _st in ENTRY_POINTS.items():
    globals()[_n] = _make_call(_n, _st)


def lc_csa_sparse_attn_workspace_bytes(args: AttnArgs) -> int:
    return int(load().lc_csa_sparse_attn_workspace_bytes(ctypes.byref(args)))


def lc_hca_attn_workspace_bytes(args: AttnArgs) -> int:
    return int(load().lc_hca_attn_workspace_bytes(ctypes.byref(args)))


def lc_hca_attn_prefill_workspace_bytes(args: AttnArgs) -> int:
    return int(load().lc_hca_attn_prefill_workspace_bytes(ctypes.byref(args)))


def lc_csa_index_topk_workspace_bytes(args: IndexTopkArgs, decode: bool) -> int:
    return int(load().lc_csa_index_topk_workspace_bytes(ctypes.byref(args), 1 if decode else 0))


def lc_csa_sparse_attn_decode_static_capacity() -> int:
    return int(load().lc_csa_sparse_attn_decode_static_capacity())


def lc_version() -> str:
    return load().lc_version().decode()
