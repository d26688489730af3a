"""GPU parity at the full workload sizes, in the launch configuration the benchmark
times.  Prefill workloads are checked on a sample of queries the oracle computes one by
one (first, last, where the visible count crosses 0 and k, and evenly spaced); decode
workloads on every sequence."""
import numpy as np
import pytest

from long_context_sparse_softmax_b200 import workloads as wl
from tests.gpu_checks import check_decode, check_prefill, save_report

pytestmark = [pytest.mark.gpu]


def sample_queries(spec: wl.Spec, n: int = 64):
    """First, last, the n_vis crossings of 1 and k, and evenly spaced queries."""
    q = set([0, spec.n_q - 1])
    for target in (1, max(spec.k, 1)):
        p = target * spec.m + spec.W - 1          # first position with n_vis == target
        for d in (-1, 0, 1):
            i = p + d - spec.q_first
            if 0 <= i < spec.n_q:
                q.add(i)
    rest = n - len(q)
    q.update(int(v) for v in np.linspace(0, spec.n_q - 1, max(rest, 2)).round())
    return sorted(q)


def test_full_csa_decode_b32_128k():
    rep = check_decode(wl.CSA_DECODE)
    save_report("full_csa_decode_b32_128k", rep)
    print(rep)


def test_full_csa_prefill_64k():
    rep = check_prefill(wl.CSA_PREFILL, q_sel=sample_queries(wl.CSA_PREFILL))
    save_report("full_csa_prefill_64k", rep)
    print(rep)


def test_full_hca_prefill_1m():
    rep = check_prefill(wl.HCA_PREFILL, q_sel=sample_queries(wl.HCA_PREFILL))
    save_report("full_hca_prefill_1m", rep)
    print(rep)


def test_full_mixed_decode_1m():
    rep = {"csa": check_decode(wl.MIXED_CSA), "hca": check_decode(wl.MIXED_HCA)}
    save_report("full_mixed_decode_1m", rep)
    print(rep)
