"""The step as a CUDA graph with its host copies (runner.capture_step with io), against the
same step launched call by call: the replay must bring every per-step input back from the
host and produce the same output and lse, bit for bit (every kernel is deterministic)."""
import pytest
import torch

from long_context_sparse_softmax_b200 import runner
from long_context_sparse_softmax_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_step_graph_with_host_copies_matches_eager_step():
    spec = wl.shrink(wl.CSA_DECODE, name="graph_io", seed=55, seq_lens=(3000, 1027, 2048), k=256)
    r = runner.Decode(wl.make_decode(spec, "cuda"), "cuda")
    main = torch.cuda.Stream()
    side = [torch.cuda.Stream() for _ in range(3)]
    torch.cuda.synchronize()
    r.step_overlapped(main, side)
    torch.cuda.synchronize()
    assert r.read_status() == 0
    ref_out, ref_lse = r.out.cpu(), r.lse.cpu()

    h2d = {st: [(d, d.cpu().pin_memory()) for d in ts] for st, ts in r.host_inputs().items()}
    d2h = [(torch.empty(d.shape, dtype=d.dtype, pin_memory=True), d) for d in r.host_outputs()]
    g = runner.capture_step([r], main, side, None, [(h2d, d2h)])
    # the replay has to restore every input from the host
    for pairs in h2d.values():
        for d, _ in pairs:
            d.zero_()
    r.out.zero_()
    r.lse.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(main):
        g.replay()
    torch.cuda.synchronize()
    assert r.read_status() == 0
    assert torch.equal(d2h[0][0], ref_out)
    assert torch.equal(d2h[1][0], ref_lse)
