"""Oracle composition of the path's stages (TEST INFRASTRUCTURE; see lc_oracle).

Each helper turns raw storage arrays into the next stage's values the way the path
does it: compute in float64, cast to the storage format the stage writes, and hand
the decoded stored values to the next stage.  Nothing here is shared with the
library; inputs are numpy arrays of raw bits and plain integers.
"""
from __future__ import annotations

from typing import Dict, Sequence

import numpy as np

from . import lc_oracle as O


def stored(fmt: int, y: np.ndarray, d_n: int):
    """Cast float64 rows to storage, and decode the stored rows back to float64."""
    x, r = O.rows_from_f64(fmt, y, d_n)
    return O.rows_to_f64(fmt, x, r), x, r


def raw_rows(fmt: int, x: np.ndarray) -> np.ndarray:
    """Raw token / query rows (FP32 or BF16 bits) as float64."""
    return O.rows_to_f64(fmt, x)


def indexer_f64(fmt: int, op: Dict[str, np.ndarray]) -> np.ndarray:
    if fmt == O.IDX_F32:
        return np.asarray(op["f32"], dtype=np.float32).astype(np.float64)
    return O.mxfp4_to_f64(op["codes"], op["scales"])


def entries_from_tokens(x, g: np.ndarray, m: int, lo: int, d_r: int, kv_fmt: int, d_n: int,
                        first_block: int = 0, n_blocks=None, tok_pos0: int = 0, chunk: int = 4096):
    """Compress complete blocks of raw token rows (float64), then cast to the entry format.

    x is a float64 array [T, D] or a callable (r0, n) -> rows r0..r0+n-1 as float64, so a
    1M-token context is converted `chunk` blocks at a time."""
    if n_blocks is None:
        n_blocks = (tok_pos0 + g.shape[0]) // m - first_block
    parts_f, parts_x, parts_r = [], [], []
    for b0 in range(0, n_blocks, chunk):
        nb = min(chunk, n_blocks - b0)
        j0 = first_block + b0
        r0 = j0 * m - tok_pos0
        xs = raw_rows_cache(x, r0, nb * m)
        y = O.compress(xs, g[r0:r0 + nb * m], m, lo, d_r, first_block=j0, tok_pos0=j0 * m, n_blocks=nb)
        f, sx, sr = stored(kv_fmt, y, d_n)
        parts_f.append(f)
        parts_x.append(sx)
        parts_r.append(sr)
    f = np.concatenate(parts_f) if parts_f else np.zeros((0, 0))
    sx = np.concatenate(parts_x) if parts_x else None
    sr = np.concatenate(parts_r) if parts_r and parts_r[0] is not None else None
    return f, sx, sr


def raw_rows_cache(x, r0: int, n: int):
    """Rows r0 .. r0+n-1 of x as float64 (x is either float64 already or a callable)."""
    if callable(x):
        return x(r0, n)
    return x[r0:r0 + n]


def visible_scores(qI: np.ndarray, kI: np.ndarray, w: np.ndarray, p: int, m: int, W_x: int):
    """Indexer scores of the entries visible to a query at p (float64) and their count."""
    n_vis = O.n_visible(p, m, W_x, kI.shape[0])
    return O.index_scores(qI, kI[:n_vis], w), n_vis


def select(qI: np.ndarray, kI: np.ndarray, w: np.ndarray, p: int, m: int, W_x: int, k: int):
    """Indexer + top-k for one query: (ascending indices, visible scores, n_vis)."""
    s, n_vis = visible_scores(qI, kI, w, p, m, W_x)
    return O.topk(s, k), s, n_vis


def padded(idx: Sequence[int], k: int) -> np.ndarray:
    out = -np.ones(k, dtype=np.int64)
    out[:len(idx)] = idx
    return out


def cast_out(o: np.ndarray, out_f32: bool) -> np.ndarray:
    """Attention output as stored: FP32, or BF16 decoded back to float64."""
    if out_f32:
        return o.astype(np.float32).astype(np.float64)
    return O.bf16_to_f64(O.f64_to_bf16(o))
