"""Seeded synthetic inputs for the CSA / HCA attention path.

This module is shared by the tests, the benchmark and the smoke check. It holds the
workload shapes and the seeded generators of their inputs, and none of the method's
arithmetic: no RMSNorm, RoPE, pooling, scoring, selection or softmax lives here.
Two pieces of input preparation do live here, because the path consumes their
output as given data:

* casts of N(0,1) draws to the storage types (torch's own casts), and
* MXFP4 encoding of the indexer keys already in a decode cache (the path quantises the
  indexer queries and the keys of new blocks itself, from raw BF16 rows).

Shapes follow the DeepSeek-V4 pages: m = 4 (CSA) and m' = 128 (HCA), a 128-token
window, top-k 512 (Flash) / 1024 (Pro), 576-dim entries with 64 RoPE dims kept in
BF16 and the rest in FP8 (page "DeepSeek-V4 论文分析", §二 model table and §8.2;
"解读 DeepSeek V4", CSA / HCA sections and "其他架构细节").

Every tensor is drawn from its own generator, seeded from (workload seed, tensor
name), so a tensor does not depend on which others were drawn before it.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, Optional, Tuple

import torch

# Storage-format identifiers (mirror the LC_FMT_* values of include/lc.h).
FMT_F32 = 0        # one FP32 array [n, D]
FMT_BF16 = 1       # one BF16 array [n, D]
FMT_E4M3_BF16 = 2  # nope dims as E4M3 [n, d_n] + RoPE dims as BF16 [n, d_r]

IDX_F32 = 0        # indexer operands in FP32
IDX_MXFP4 = 3      # indexer operands in MXFP4 (E2M1 codes + E8M0 scale per 32)


@dataclasses.dataclass(frozen=True)
class Spec:
    """One workload shape.

    kind: "csa_prefill" | "csa_decode" | "hca_prefill" | "hca_decode".
    Prefill: one sequence of ``seq_lens[0]`` tokens; queries at positions
    ``q_first .. q_first + n_q - 1``.  Decode: one query per sequence at position
    ``L_b - 1``.
    """
    name: str
    kind: str
    seed: int
    seq_lens: Tuple[int, ...]
    D: int = 576
    d_r: int = 64
    rope_off: int = 512      # first RoPE dim inside a row (single-array formats)
    H: int = 64
    m: int = 4
    W: int = 128
    k: int = 512
    H_I: int = 64
    d_I: int = 128
    fp32: bool = False       # tiny correctness case: every tensor FP32
    q_bf16: bool = False     # prepped queries kept as BF16 (HCA prefill)
    q_first: int = 0
    n_q: int = 0
    overlap: bool = False    # window/compressed overlap reading (W_x = 0)
    ring: bool = True        # decode: each sequence's window rows are a ring of W rows
    w_per_query: bool = False  # indexer head weights per query [n_q, H_I] instead of shared [H_I]
    v_nope: bool = False     # values are the non-RoPE dims of the entries (outputs D - d_r dims)
    out32: bool = False      # FP32 attention outputs with the narrow input formats

    @property
    def d_n(self) -> int:
        return self.D - self.d_r

    @property
    def Dv(self) -> int:
        """Dims of each head's output: the value rows' dims."""
        return self.D - self.d_r if self.v_nope else self.D

    @property
    def scale(self) -> float:
        return 1.0 / float(self.D) ** 0.5

    @property
    def raw_fmt(self) -> int:
        return FMT_F32 if self.fp32 else FMT_BF16

    @property
    def kv_fmt(self) -> int:
        return FMT_F32 if self.fp32 else FMT_E4M3_BF16

    @property
    def q_fmt(self) -> int:
        if self.fp32:
            return FMT_F32
        return FMT_BF16 if self.q_bf16 else FMT_E4M3_BF16

    @property
    def win_fmt(self) -> int:
        return FMT_F32 if self.fp32 else FMT_BF16

    @property
    def idx_fmt(self) -> int:
        return IDX_F32 if self.fp32 else IDX_MXFP4

    @property
    def out_f32(self) -> bool:
        return self.fp32 or self.out32

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def is_decode(self) -> bool:
        return self.kind.endswith("decode")

    @property
    def is_csa(self) -> bool:
        return self.kind.startswith("csa")

    def n_entries(self, L: int) -> int:
        """Stored compressed entries for a context of L tokens: complete blocks only."""
        return L // self.m


def _cfg5_lengths() -> Tuple[int, ...]:
    g = torch.Generator().manual_seed(4)
    return tuple(int(v) for v in torch.randint(524288, 1048576 + 1, (8,), generator=g))


# The five workloads.  Seeds 1-3 are not fixed by the workload statements and are
# chosen here; ragged lengths of the mixed decode are drawn with seed 4.
TINY_CSA_PREFILL = Spec("tiny_csa_prefill_f32_L1024", "csa_prefill", 0, (1024,), D=128, d_r=64,
                        rope_off=0, H=8, m=4, W=128, k=64, H_I=4, d_I=64, fp32=True,
                        q_first=0, n_q=1024)
CSA_DECODE = Spec("csa_decode_b32_L131072_k512", "csa_decode", 1, (131072,) * 32, H=64, m=4, k=512)
HCA_PREFILL = Spec("hca_prefill_L1048576_q4096", "hca_prefill", 2, (1 << 20,), H=64, m=128, k=0,
                   q_bf16=True, q_first=(1 << 20) - 4096, n_q=4096)
CSA_PREFILL = Spec("csa_prefill_L65536_k1024_h128", "csa_prefill", 3, (65536,), H=128, m=4, k=1024,
                   q_first=0, n_q=65536)
MIXED_CSA = Spec("mixed_decode_csa_b8_1M_k1024", "csa_decode", 4, _cfg5_lengths(), H=64, m=4, k=1024)
MIXED_HCA = Spec("mixed_decode_hca_b8_1M", "hca_decode", 4, _cfg5_lengths(), H=64, m=128, k=0)

WORKLOADS = {
    "tiny_csa_prefill": (TINY_CSA_PREFILL,),
    "csa_decode": (CSA_DECODE,),
    "hca_prefill": (HCA_PREFILL,),
    "csa_prefill": (CSA_PREFILL,),
    "mixed_decode": (MIXED_CSA, MIXED_HCA),
}


# ---------------------------------------------------------------------------------
# seeded draws
# ---------------------------------------------------------------------------------
def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1000003 + zlib.crc32(name.encode())) & 0x7FFFFFFFFFFFFFFF)
    return g


def randn(seed: int, name: str, shape, device) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(seed, name, device), device=device, dtype=torch.float32)


def rand(seed: int, name: str, shape, device) -> torch.Tensor:
    return torch.rand(shape, generator=_gen(seed, name, device), device=device, dtype=torch.float32)


def to_bf16_bits(x: torch.Tensor) -> torch.Tensor:
    """torch's round-to-nearest-even cast to BF16, returned as raw int16 bits."""
    return x.to(torch.bfloat16).view(torch.int16)


def to_e4m3_bits(x: torch.Tensor) -> torch.Tensor:
    """torch's cast to E4M3 (inputs are N(0,1), far inside the +-448 range)."""
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


_E2M1_MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def mxfp4_encode(v: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Encode FP32 values [..., d] as MXFP4 (OCP Microscaling Formats v1.0).

    Per block of 32 along the last axis: shared scale X = 2^(floor(log2 amax) - 2)
    (E8M0 code X + 127; an all-zero block gets X = 1), elements v / X rounded to the
    nearest E2M1 value (ties to the even code), saturating at +-6.
    Returns (codes uint8 [..., d/2] with element 2i in the low nibble and 2i+1 in the
    high nibble, scales uint8 [..., d/32]).
    """
    d = v.shape[-1]
    assert d % 32 == 0
    blocks = v.float().reshape(*v.shape[:-1], d // 32, 32)
    amax = blocks.abs().amax(-1)
    # floor(log2 amax) taken exactly from the binary exponent (frexp: amax = f * 2^e, f in [0.5, 1))
    _, ex = torch.frexp(torch.where(amax > 0, amax, torch.ones_like(amax)))
    e = torch.where(amax > 0, (ex - 1 - 2).float(), torch.zeros_like(amax)).clamp(-127, 127)
    scaled = blocks / torch.exp2(e).unsqueeze(-1)
    a = scaled.abs().clamp(max=6.0)
    mids = torch.tensor(_E2M1_MIDS, device=v.device, dtype=torch.float32)
    lo = torch.bucketize(a, mids, right=False)   # ties go to the smaller code
    hi = torch.bucketize(a, mids, right=True)    # ties go to the larger code
    code = torch.where((lo != hi) & (hi % 2 == 0), hi, lo)
    code = code | ((scaled < 0) & (code > 0)).to(code.dtype) << 3
    code = code.to(torch.uint8).reshape(*v.shape[:-1], d)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    scales = (e + 127).to(torch.uint8)
    return packed.contiguous(), scales.contiguous()


def _indexer_operand(spec: Spec, name: str, shape, device) -> Dict[str, torch.Tensor]:
    v = randn(spec.seed, name, shape, device)
    if spec.idx_fmt == IDX_F32:
        return {"f32": v.contiguous()}
    codes, scales = mxfp4_encode(v)
    return {"codes": codes, "scales": scales}


def _i32(vals, device) -> torch.Tensor:
    return torch.tensor(list(vals), dtype=torch.int32, device=device)


def _i64(vals, device) -> torch.Tensor:
    return torch.tensor(list(vals), dtype=torch.int64, device=device)


def _synthetic_cache(spec: Spec, n_rows: int, name: str, device) -> Dict[str, torch.Tensor]:
    """Cached compressed entries drawn directly: N(0,1) per dim in the storage format."""
    v = randn(spec.seed, name, (n_rows, spec.D), device)
    if spec.kv_fmt == FMT_F32:
        return {"x": v}
    return {"x": to_e4m3_bits(v[:, :spec.d_n]).contiguous(),
            "rope": to_bf16_bits(v[:, spec.d_n:]).contiguous()}


def _raw_rows(spec: Spec, name: str, shape, device) -> torch.Tensor:
    v = randn(spec.seed, name, shape, device)
    return v if spec.raw_fmt == FMT_F32 else to_bf16_bits(v)


# ---------------------------------------------------------------------------------
# workload inputs
# ---------------------------------------------------------------------------------
def make_prefill(spec: Spec, device="cpu") -> Dict[str, object]:
    """One sequence, raw tokens given; entries and window rows are computed by the path.

    Tensors: x [L, D] raw token KV, g [L] gate logits, q_raw [n_q, H, D], the
    indexer rows (CSA; MXFP4 workloads: raw BF16 qI_raw [n_q, H_I, d_I] and per-token
    kI_raw [L, d_I], which the path quantises and pools; FP32: qI and kI [n_c, d_I]
    given directly), w [H_I], sink [H].
    """
    (L,) = spec.seq_lens
    s = spec
    out: Dict[str, object] = {"spec": s, "L": L}
    out["x"] = _raw_rows(s, "x", (L, s.D), device)
    out["g"] = randn(s.seed, "g", (L,), device)
    out["q_raw"] = _raw_rows(s, "q", (s.n_q, s.H, s.D), device)
    out["sink"] = randn(s.seed, "sink", (s.H,), device)
    n_c = s.n_entries(L)
    out["n_c"] = n_c
    if s.is_csa:
        if s.idx_fmt == IDX_MXFP4:
            # raw indexer rows: the path quantises the queries and pools + quantises the
            # keys of every complete block itself
            out["qI_raw"] = to_bf16_bits(randn(s.seed, "qI", (s.n_q, s.H_I, s.d_I), device))
            out["kI_raw"] = to_bf16_bits(randn(s.seed, "kI", (L, s.d_I), device))
        else:
            out["qI"] = _indexer_operand(s, "qI", (s.n_q, s.H_I, s.d_I), device)
            out["kI"] = _indexer_operand(s, "kI", (n_c, s.d_I), device)
        out["w"] = rand(s.seed, "w", (s.n_q, s.H_I) if s.w_per_query else (s.H_I,), device)
    # positions and the batch descriptor (one sequence)
    q_pos = torch.arange(s.q_first, s.q_first + s.n_q, dtype=torch.int32, device=device)
    out["q_pos"] = q_pos
    # window rows: the raw tokens the queries can reach, prepped with H = 1
    w0 = max(0, s.q_first - s.W + 1) if s.W > 0 else s.q_first
    out["win_pos0"] = w0
    out["win_pos"] = torch.arange(w0, s.q_first + s.n_q, dtype=torch.int32, device=device)
    out["batch"] = {
        "q_start": _i32([0, s.n_q], device),
        "q_pos0": _i32([s.q_first], device),
        "ent_start": _i64([0], device),
        "n_ent": _i32([n_c], device),
        "win_start": _i64([0], device),
        "win_pos0": _i32([w0], device),
        "win_len": _i32([s.q_first + s.n_q - w0], device),
    }
    return out


def make_decode(spec: Spec, device="cpu") -> Dict[str, object]:
    """B sequences, one query each at p = L_b - 1, on an existing cache.

    Cache tensors are drawn directly in their storage formats: compressed entries
    (nope E4M3 + RoPE BF16, or FP32), prepped window rows [B*W, D] for positions
    L_b - W .. L_b - 1 (BF16 or FP32; with spec.ring a ring buffer of W rows per
    sequence, position t in row b W + t mod W), indexer keys kI [sum n_c, d_I].  The newest
    block's raw tokens (x_tail [B, m, D], g_tail [B, m]) and the newest token's raw
    row x_new [B, D] feed the decode-time compression and window preparation.  MXFP4
    workloads give the query's raw indexer rows (qI_raw [B, H_I, d_I] BF16) and the
    newest block's raw indexer-key rows (kI_tail [B, m, d_I] BF16) for the step to
    quantise and pool.
    """
    s = spec
    B = s.num_seqs
    n_c = [s.n_entries(L) for L in s.seq_lens]
    ent_start = [0]
    for n in n_c[:-1]:
        ent_start.append(ent_start[-1] + n)
    tot = sum(n_c)
    out: Dict[str, object] = {"spec": s, "n_c": n_c}
    out["cache"] = _synthetic_cache(s, tot, "cache", device)
    win_rows = B * s.W
    wv = randn(s.seed, "win", (win_rows, s.D), device)   # row b W + i: position win_pos0[b] + i
    if s.ring:
        # ring buffer of W rows per sequence: position t in slot t mod W
        slot = torch.tensor([b * s.W + (max(0, L - s.W) + i) % s.W for b, L in enumerate(s.seq_lens)
                             for i in range(s.W)], dtype=torch.int64, device=device)
        ring = torch.empty_like(wv)
        ring[slot] = wv
        wv = ring
    out["win"] = wv if s.win_fmt == FMT_F32 else to_bf16_bits(wv)
    out["q_raw"] = _raw_rows(s, "q", (B, s.H, s.D), device)
    out["x_new"] = _raw_rows(s, "x_new", (B, s.D), device)
    out["x_tail"] = _raw_rows(s, "x_tail", (B, s.m, s.D), device)
    out["g_tail"] = randn(s.seed, "g_tail", (B, s.m), device)
    out["sink"] = randn(s.seed, "sink", (s.H,), device)
    if s.is_csa:
        if s.idx_fmt == IDX_MXFP4:
            # the step quantises the query's raw indexer rows and pools + quantises the
            # indexer key of the block the newest token closed
            out["qI_raw"] = to_bf16_bits(randn(s.seed, "qI", (B, s.H_I, s.d_I), device))
            out["kI_tail"] = to_bf16_bits(randn(s.seed, "kI_tail", (B, s.m, s.d_I), device))
        else:
            out["qI"] = _indexer_operand(s, "qI", (B, s.H_I, s.d_I), device)
        out["kI"] = _indexer_operand(s, "kI", (tot, s.d_I), device)
        out["w"] = rand(s.seed, "w", (B, s.H_I) if s.w_per_query else (s.H_I,), device)
    out["q_pos"] = _i32([L - 1 for L in s.seq_lens], device)
    out["batch"] = {
        "q_start": _i32(range(B + 1), device),
        "q_pos0": _i32([L - 1 for L in s.seq_lens], device),
        "ent_start": _i64(ent_start, device),
        "n_ent": _i32(n_c, device),
        "win_start": _i64([b * s.W for b in range(B)], device),
        "win_pos0": _i32([max(0, L - s.W) for L in s.seq_lens], device),
        "win_len": _i32([min(s.W, L) for L in s.seq_lens], device),
        "win_ring": s.W if s.ring and s.W > 0 else 0,
    }
    # the newest block completes at the current token only when m divides L_b
    out["blk_count"] = _i32([1 if L % s.m == 0 else 0 for L in s.seq_lens], device)
    out["blk_first"] = _i32([max(0, L // s.m - 1) for L in s.seq_lens], device)
    return out


def shrink(spec: Spec, **kw) -> Spec:
    """A smaller variant of a workload (same formats), for oracle-sized tests."""
    return dataclasses.replace(spec, **kw)


def cpu_numpy(t: Optional[torch.Tensor]):
    """Host numpy copy of a tensor (raw bits for int16/uint8 storage)."""
    if t is None:
        return None
    return t.detach().cpu().numpy()
