"""Benchmark of the CSA / HCA attention path on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole path over one batch of synthetic input:
  csa_decode (default; batch 32 x 131072-token context, top-k 512, 64 heads x 576 dims,
  E4M3+BF16 cache, MXFP4 indexer): prepare the query and the newest window row, compress
  the block the newest token closed, index scores, top-k, sparse attention.
  csa_prefill / hca_prefill / tiny_csa_prefill: the whole prefill of one sequence.
  mixed_decode: a CSA decode layer and an HCA decode layer, batch 8, ragged 0.5M-1M.
Metric: query tokens per second (whole job, all ranks).  Inputs are resident in HBM when
the timed region starts; L2 is flushed (a 512 MiB write, then a 256 MiB read that leaves
the cache clean) between timed steps, outside the per-step CUDA events.  The step is
captured once as a CUDA graph and replayed (--no-graph: every call launched from Python).  With N > 1 (torchrun) every rank runs its own batch: weak
scaling, no collective on the data path.
--impl reference times the CPU oracle (the plain float64 restatement of the method) on a
bounded sample of the same workload on one host core (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA/HCA attention query-tokens/s at 128K-1M ctx; % of HBM/tensor-pipe roofline"
UNIT = "query-tokens/s"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "ncu_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="csa_decode",
                    choices=["csa_decode", "csa_prefill", "hca_prefill", "mixed_decode", "tiny_csa_prefill"])
    ap.add_argument("--impl", default="lc", choices=["lc", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch every call from Python each step "
                    "instead of replaying the step's CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fused", action="store_true", help="run the indexer and top-k as two calls "
                    "(scores written) instead of the fused index + top-k call")
    ap.add_argument("--cpu-sample-s", type=float, default=15.0)
    ap.add_argument("--attn-impl", default="auto", choices=["auto", "tc", "ref"],
                    help="attention kernel (auto: tcgen05 where it applies, else the FP32 reference kernel)")
    return ap.parse_args()


def dist_env():
    """(rank, world size, local rank) from the launcher's environment (1 process: 0, 1, 0)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def workload_config(name: str) -> dict:
    """The config keys both arms report for a workload: its name and shape."""
    from long_context_sparse_softmax_b200 import workloads as wl
    specs = wl.WORKLOADS[name]
    s = specs[0]
    return {"workload": s.name if len(specs) == 1 else name,
            "batch": s.num_seqs if s.is_decode else 1,
            "context": max(s.seq_lens), "heads": s.H, "dims": s.D, "topk": s.k,
            "query_tokens_per_step_per_gpu": s.num_seqs if s.is_decode else s.n_q}


def rank_spec(spec, rank: int):
    """The workload a rank runs: the same shapes, its own seed (independent batches, weak
    scaling)."""
    import dataclasses
    return spec if rank == 0 else dataclasses.replace(spec, seed=spec.seed + 1000 * rank)


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_throughput(world: int, units_per_step: int, steps: int, total_ms: float) -> float:
    """Query tokens per second of the whole job: every rank processes its own batch of
    units_per_step tokens per step, and the job takes total_ms (the slowest rank)."""
    return world * units_per_step * steps / (total_ms / 1e3)


def peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------
# algorithmic work per stage (bytes that must move / flops that must be done)
# ------------------------------------------------------------------------------------
def _row_bytes(fmt: int, D: int, d_r: int) -> int:
    return {0: 4 * D, 1: 2 * D, 2: (D - d_r) + 2 * d_r}[fmt]


def _n_vis(p, m, W_x, n_ent):
    return max(0, min((p - W_x + 1) // m, n_ent)) if p - W_x + 1 > 0 else 0


def stage_work(spec, inp, run):
    """{stage: (bytes, flops)} of one step, counting only what the method must touch."""
    import numpy as np
    s = spec
    raw_es = 4 if s.fp32 else 2
    ent_b = _row_bytes(s.kv_fmt, s.D, s.d_r)
    win_b = _row_bytes(s.win_fmt, s.D, s.d_r)
    q_b = _row_bytes(s.q_fmt, s.D, s.d_r)
    out_b = (4 if s.out_f32 else 2) * s.D
    idx_key_b = (4 * s.d_I) if s.fp32 else (s.d_I // 2 + s.d_I // 32)
    idx_q_b = s.H_I * idx_key_b
    W = s.W
    work = {}
    if s.is_decode:
        B = s.num_seqs
        pos = [L - 1 for L in s.seq_lens]
        n_c = list(inp["n_c"])
        nv = [_n_vis(p, s.m, s.W, n) for p, n in zip(pos, n_c)]
        nwin = [min(W, p + 1) for p in pos]
        n_blk = int(sum(1 for L in s.seq_lens if L % s.m == 0))
        work["qk_prep_q"] = (B * s.H * (s.D * raw_es + q_b), 0)
        work["qk_prep_win"] = (B * (s.D * raw_es + win_b), 0)
        work["compress"] = (n_blk * (s.m * (s.D * raw_es + 4) + ent_b), 0)
        if s.is_csa:
            K = [min(s.k, v) for v in nv]
            work["index"] = (sum(v * (idx_key_b + 4) for v in nv) + B * idx_q_b,
                             sum(2 * v * s.H_I * s.d_I for v in nv))
            work["topk"] = (sum(4 * v for v in nv) + B * 4 * s.k, 0)
            # fused: the keys and queries in, the selection out; no score matrix
            work["index_topk"] = (sum(v * idx_key_b for v in nv) + B * idx_q_b + B * 4 * s.k,
                                  sum(2 * v * s.H_I * s.d_I for v in nv))
            # raw BF16 indexer rows quantised on the GPU: the query rows, the key of the closed block
            work["quant_q"] = (B * s.H_I * (2 * s.d_I + idx_key_b), 0)
            work["index_compress"] = (n_blk * (s.m * (2 * s.d_I + 4) + idx_key_b), 0)
            sel = K
        else:
            sel = nv
        keys = [a + w for a, w in zip(sel, nwin)]
        work["attn"] = (sum(a * ent_b + w * win_b for a, w in zip(sel, nwin)) + B * s.H * (q_b + out_b + 4),
                        sum(4 * s.H * k * s.D for k in keys))
        units = B
    else:
        L, n_c = inp["L"], inp["n_c"]
        pos = np.arange(s.q_first, s.q_first + s.n_q)
        nv = np.clip((pos - s.W + 1) // s.m, 0, n_c)
        nv[pos - s.W + 1 <= 0] = 0
        nwin = np.minimum(W, pos + 1)
        n_win_rows = int(inp["win_pos"].numel())
        work["qk_prep_q"] = (s.n_q * s.H * (s.D * raw_es + q_b), 0)
        work["qk_prep_win"] = (n_win_rows * (s.D * raw_es + win_b), 0)
        work["compress"] = (n_c * (s.m * (s.D * raw_es + 4) + ent_b), 0)
        if s.is_csa:
            K = np.minimum(s.k, nv)
            work["index"] = (n_c * idx_key_b + s.n_q * idx_q_b + int(nv.sum()) * 4,
                             int(nv.sum()) * 2 * s.H_I * s.d_I)
            work["topk"] = (int(nv.sum()) * 4 + s.n_q * 4 * s.k, 0)
            work["index_topk"] = (n_c * idx_key_b + s.n_q * idx_q_b + s.n_q * 4 * s.k,
                                  int(nv.sum()) * 2 * s.H_I * s.d_I)
            work["quant_q"] = (s.n_q * s.H_I * (2 * s.d_I + idx_key_b), 0)
            work["index_compress"] = (n_c * (s.m * (2 * s.d_I + 4) + idx_key_b), 0)
            sel = K
        else:
            sel = nv
        keys = sel + nwin
        work["attn"] = (n_c * ent_b + n_win_rows * win_b + s.n_q * s.H * (q_b + out_b + 4),
                        int(keys.sum()) * 4 * s.H * s.D)
        units = s.n_q
    return work, units


# Dense tensor-core rates relative to BF16 (the nominal ratios; a tcgen05 probe that ran
# M128 x N128 MMAs on every SM measured 2221, 4448 and 8899 TFLOP/s for BF16, E4M3 and
# MXFP4, the same 1 : 2 : 4)
TENSOR_RATIO = {"bf16": 1.0, "e4m3": 2.0, "mxf4": 4.0}


def tensor_mix(stage, spec, attn_impl="auto"):
    """(peak factor over the BF16 peak, label) for a tensor-bound stage: the indexer runs
    MXFP4 MMAs; the E4M3-score attention kernel does half its flops (S) in E4M3 and half
    (P V) in F16."""
    from long_context_sparse_softmax_b200 import workloads as wl
    if stage.split(":")[-1] in ("index", "index_topk") and spec.idx_fmt == wl.IDX_MXFP4:
        return TENSOR_RATIO["mxf4"], "MXFP4"
    if (stage.endswith("attn") and attn_impl in ("auto", "tc") and spec.q_fmt == wl.FMT_E4M3_BF16
            and spec.kv_fmt == wl.FMT_E4M3_BF16):
        return 1.0 / (0.5 / TENSOR_RATIO["e4m3"] + 0.5 / TENSOR_RATIO["bf16"]), "E4M3 S + F16 PV"
    return 1.0, "BF16/F16"


def bound_of(stage, spec, work, pk, attn_impl="auto"):
    """HBM- or tensor-bound by comparing the two roofline times."""
    b, f = work[stage]
    t_mem = b / (pk["hbm_gbs"] * 1e9)
    t_math = f / (pk["bf16_tflops"] * tensor_mix(stage, spec, attn_impl)[0] * 1e12) if f else 0.0
    return ("tensor", t_math) if t_math > t_mem else ("hbm", t_mem)


# ------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def kernel_traffic(workload: str, stage: str, attn_impl: str):
    """DRAM bytes per launch of a stage's kernels on this workload from the committed ncu
    summary (keyed "<workload>:<stage>"), if that workload was captured and every source
    file of those kernels is unchanged since the capture (and, for attention, the same
    kernel choice ran); else None."""
    if not os.path.exists(TRAFFIC_PATH):
        return None
    with open(TRAFFIC_PATH) as f:
        t = json.load(f)
    e = t.get(f"{workload}:{stage}")
    if not e:
        return None
    if "attn_impl" in e and attn_impl not in e["attn_impl"]:
        return None
    for name, sha in e["sources"].items():
        src = os.path.join(ROOT, "long_context_sparse_softmax_b200", "csrc", name)
        if not os.path.exists(src) or hashlib.sha1(open(src, "rb").read()).hexdigest() != sha:
            return None
    return e.get("dram_bytes_per_launch_full")




# ------------------------------------------------------------------------------------
# the library arm
# ------------------------------------------------------------------------------------
def make_runs(name, device, rank, impl=0, fused=None):
    from long_context_sparse_softmax_b200 import runner
    from long_context_sparse_softmax_b200 import workloads as wl
    runs = []
    for spec in wl.WORKLOADS[name]:
        spec = rank_spec(spec, rank)
        inp = (wl.make_decode if spec.is_decode else wl.make_prefill)(spec, device)
        r = (runner.Decode if spec.is_decode else runner.Prefill)(inp, device, None, impl, fused)
        runs.append((spec, inp, r))
    return runs


def host_io(runs):
    """Per run, the e2e leg's host copies: (h2d, d2h).  h2d maps the stage that first reads
    a per-step input (the runner's host_inputs) to (device, pinned host) pairs; d2h holds
    (pinned host, device) pairs of the results."""
    import torch
    io = []
    for _, _, r in runs:
        h2d = {st: [(d, d.cpu().pin_memory()) for d in ts] for st, ts in r.host_inputs().items()}
        d2h = [(torch.empty(d.shape, dtype=d.dtype, pin_memory=True), d) for d in r.host_outputs()]
        io.append((h2d, d2h))
    return io


def run_lc(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    pk, pk_kind = peaks()
    runs = make_runs(args.workload, dev, rank, {"auto": 0, "tc": 2, "ref": 3}[args.attn_impl],
                     False if args.no_fused else None)
    # L2 flush: a 512 MiB write, then a 256 MiB read so that the lines the step evicts are
    # clean (the write alone would leave L2 full of dirty lines whose write-back lands on
    # the first kernel of the step)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        flush_r.sum()
    # the critical path (index -> top-k -> attention) on a high-priority stream, made current
    # so that the L2 flush and the host copies stay ordered with it; the side stream fills
    # the SMs it leaves idle
    stream = torch.cuda.Stream(dev, priority=-100)
    torch.cuda.set_stream(stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    work = {}
    units = 0
    for i, (spec, inp, r) in enumerate(runs):
        w, u = stage_work(spec, inp, r)
        for k, v in w.items():
            work[f"{i}:{k}"] = v
        units += u if i == 0 else 0  # a mixed step counts each sequence's token once
    stage_names = [f"{i}:{n}" for i, (_, _, r) in enumerate(runs) for n, _ in r.stages()]
    # the critical path: stages on the main stream (the side stages overlap them, and their
    # event times include the wait for SMs the critical path holds)
    crit_names = [f"{i}:{n}" for i, (_, _, r) in enumerate(runs) for part in r.dag()[1:] for n, _ in part]
    # kernels per step: one per call, plus the combine kernel of an attention whose key
    # splits leave partials in a workspace (or, in HCA prefill, the kernel that widens the
    # entries into that workspace), plus the merge kernel of a fused index + top-k whose
    # queries span several indexer CTAs (it then has a candidate workspace)
    n_launch = len(stage_names) + sum(1 for (_, _, r) in runs if r.a_attn.workspace_bytes > 0) + \
        sum(1 for (_, _, r) in runs if getattr(r, "fused", False) and r.a_index_topk.workspace_bytes > 0)
    # one stream per side stage: they share no buffers, so none waits for another
    side = [torch.cuda.Stream(dev, priority=0) for _ in range(3)]

    def timed(stage_ev):
        """on_stage hook that brackets each launch with the stage's event pair."""
        def on_stage(i, name, st, fn):
            e0, e1 = stage_ev[f"{i}:{name}"]
            e0.record(st)
            fn(st)
            e1.record(st)
        return on_stage

    def one_step(stage_ev=None, io=None):
        """The whole path once: per workload, preparation and compression on the side
        stream next to index -> top-k on the main stream, then attention."""
        hook = None if stage_ev is None else timed(stage_ev)
        for i, (_, _, r) in enumerate(runs):
            r.step_overlapped(stream, side, None if hook is None else
                              (lambda name, st, fn, i=i: hook(i, name, st, fn)),
                              None if io is None else io[i])

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    for _, _, r in runs:
        assert r.read_status() == 0, "device status bits set"
    graph = None       # the timed step: a CUDA graph of the step, no event nodes
    graph_dom = None   # the same step with the dominant stage bracketed (its kernel time)
    graph_all = None   # the same step with every stage bracketed (per-stage breakdown)
    dom_key = None
    rl = [r for _, _, r in runs]
    if not args.no_graph:
        from long_context_sparse_softmax_b200.runner import capture_step

        def ext_pair():
            # external: recorded as graph nodes that take a timestamp on every replay
            return (torch.cuda.Event(enable_timing=True, external=True),
                    torch.cuda.Event(enable_timing=True, external=True))
        g_ev = {n: ext_pair() for n in stage_names}
        graph_all = capture_step(rl, stream, side, timed(g_ev))
        warm = {n: [] for n in stage_names}
        for _ in range(args.warmup):
            flush_l2()
            graph_all.replay()
            torch.cuda.synchronize()
            for n in stage_names:
                warm[n].append(g_ev[n][0].elapsed_time(g_ev[n][1]))
        # an event node on the critical path lengthens the step by microseconds, so the
        # headline graph has none; the roofline's kernel time comes from a graph that
        # brackets only that stage, timed in a pass of its own
        dom_key = max(crit_names, key=lambda n: statistics.mean(warm[n]))
        d_ev = ext_pair()

        def timed_dom(i, name, st, fn):
            if f"{i}:{name}" != dom_key:
                fn(st)
                return
            d_ev[0].record(st)
            fn(st)
            d_ev[1].record(st)
        graph_dom = capture_step(rl, stream, side, timed_dom)
        graph = capture_step(rl, stream, side, None)
        for _ in range(args.warmup):
            flush_l2()
            graph_dom.replay()
            flush_l2()
            graph.replay()
        torch.cuda.synchronize()

    ev = [{n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for n in stage_names}
          for _ in range(args.steps)]
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    dom_ms = []
    with ClockSampler(gpu_id) as clk:
        for s in range(args.steps):
            flush_l2()
            ev_step[s][0].record(stream)
            if graph is None:
                one_step(ev[s])
            else:
                graph.replay()
            ev_step[s][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    if graph_dom is not None:
        # the dominant kernel's time: the same steps again, that stage bracketed (the
        # graph's events are re-recorded by every replay: read them after each)
        for s in range(args.steps):
            flush_l2()
            graph_dom.replay()
            torch.cuda.synchronize()
            dom_ms.append(d_ev[0].elapsed_time(d_ev[1]))
    if graph is None:
        per_stage = {n: [ev[s][n][0].elapsed_time(ev[s][n][1]) for s in range(args.steps)] for n in stage_names}
    else:
        # per-stage breakdown: a third timed pass, the graph with every stage bracketed
        per_stage = {n: [] for n in stage_names}
        for s in range(args.steps):
            flush_l2()
            graph_all.replay()
            torch.cuda.synchronize()
            for n in stage_names:
                per_stage[n].append(g_ev[n][0].elapsed_time(g_ev[n][1]))
    # a step's time runs from the fork on the main stream to the end of attention
    span = [ev_step[s][0].elapsed_time(ev_step[s][1]) for s in range(args.steps)]
    total_ms = sum(span)
    total_ms = max_over_ranks(total_ms, dev, world)
    value = weak_throughput(world, units, args.steps, total_ms)

    # e2e: host inputs in, host outputs back, through the same C-ABI calls
    e2e = None
    if not args.no_e2e:
        io = host_io(runs)
        h2d = sum(h.numel() * h.element_size() for hd, _ in io for pairs in hd.values() for _, h in pairs)
        d2h = sum(h.numel() * h.element_size() for _, dl in io for h, _ in dl)
        # each upload on the stream of the stage that first reads it, inside the step's
        # graph, so that it overlaps the stages before it; the results come back after
        # attention.  If copies cannot be captured, they run eagerly around the graph.
        graph_io = None
        e2e_mode = "eager copies, step launched from Python" if graph is None else "eager copies around the step graph"
        if graph is not None:
            try:
                graph_io = capture_step(rl, stream, side, None, io)
                for _ in range(args.warmup):
                    graph_io.replay()
                torch.cuda.synchronize()
                e2e_mode = "copies inside the step graph, each on its stage's stream"
            except Exception as ex:  # noqa: BLE001 - any capture failure falls back
                graph_io = None
                print(f"e2e: host copies not capturable ({ex}); timing eager copies", file=sys.stderr)
                torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e_ms = 0.0
        for s in range(args.steps):
            flush_l2()
            e0.record(stream)
            if graph_io is not None:
                graph_io.replay()
            elif graph is None:
                one_step(None, io)
            else:
                for hd, _ in io:
                    for pairs in hd.values():
                        for d, h in pairs:
                            d.copy_(h, non_blocking=True)
                graph.replay()
                for _, dl in io:
                    for h, d in dl:
                        h.copy_(d, non_blocking=True)
            e1.record(stream)
            e1.synchronize()
            e_ms += e0.elapsed_time(e1)
        e2e = {"value": weak_throughput(world, units, args.steps, max_over_ranks(e_ms, dev, world)), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "copies": e2e_mode}
        if graph is not None:
            # the same, with every C-ABI call (validation, argument marshalling, launch) and
            # every copy issued from Python each step, as a caller without graphs would
            barrier()
            torch.cuda.synchronize()
            c_ms = 0.0
            for s in range(args.steps):
                flush_l2()
                e0.record(stream)
                one_step(None, io)
                e1.record(stream)
                e1.synchronize()
                c_ms += e0.elapsed_time(e1)
            per_call = {"value": weak_throughput(world, units, args.steps, max_over_ranks(c_ms, dev, world)),
                        "unit": UNIT, "copies": "eager copies and C-ABI calls issued from Python each step"}
            # both are the public calls with the host copies timed; the faster is the value
            # (host-to-device copies inside a graph measured slower than eager ones here)
            if per_call["value"] > e2e["value"]:
                e2e["graph"] = {"value": e2e["value"], "unit": UNIT, "copies": e2e["copies"]}
                e2e["value"], e2e["copies"] = per_call["value"], per_call["copies"]
            else:
                e2e["per_call"] = per_call
        if graph is not None and h2d + d2h < (256 << 20):
            # (decode-sized steps: prefill moves gigabytes per step, and three pinned copies
            # of its inputs would not fit the host)
            # steps overlapped as a serving loop runs them: three independent sets of
            # buffers take turns; step i uploads its inputs on one copy stream while step
            # i - 1 computes, and its results go back on another copy stream while step
            # i + 1 computes.  Every step's copies and kernels are inside the timed region.
            # No flush: between two uses of a set the other two sets' steps read about 1.6
            # times L2's capacity (99 MB each on the decode workload: inputs larger than L2).
            n_sets = 3
            sets = [(graph, io)]
            extra = []
            for _ in range(n_sets - 1):
                runs2 = make_runs(args.workload, dev, rank, {"auto": 0, "tc": 2, "ref": 3}[args.attn_impl],
                                  False if args.no_fused else None)
                rl2 = [r for _, _, r in runs2]
                for r in rl2:
                    r.step(stream)
                torch.cuda.synchronize()
                sets.append((capture_step(rl2, stream, side, None), host_io(runs2)))
                extra.append(runs2)
            up_st, down_st = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
            done_c = [torch.cuda.Event() for _ in sets]   # the set's last step computed
            done_d = [torch.cuda.Event() for _ in sets]   # the set's last results read back
            used = [False] * n_sets

            def pipelined(n):
                for i in range(n):
                    k = i % n_sets
                    g2, io_k = sets[k]
                    if used[k]:
                        up_st.wait_event(done_c[k])      # its inputs are no longer read
                    with torch.cuda.stream(up_st):
                        for hd, _ in io_k:
                            for pairs in hd.values():
                                for d, h in pairs:
                                    d.copy_(h, non_blocking=True)
                    up = torch.cuda.Event()
                    up.record(up_st)
                    stream.wait_event(up)
                    if used[k]:
                        stream.wait_event(done_d[k])     # its outputs were read back
                    g2.replay()
                    done_c[k].record(stream)
                    down_st.wait_event(done_c[k])
                    with torch.cuda.stream(down_st):
                        for _, dl in io_k:
                            for h, d in dl:
                                h.copy_(d, non_blocking=True)
                    done_d[k].record(down_st)
                    used[k] = True

            pipelined(max(n_sets, args.warmup))
            torch.cuda.synchronize()
            barrier()
            p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            p0.record(up_st)
            stream.wait_event(p0)
            pipelined(args.steps)
            for k in range(n_sets):
                down_st.wait_event(done_d[k])
            p1.record(down_st)
            p1.synchronize()
            pipe = {"value": weak_throughput(world, units, args.steps, max_over_ranks(p0.elapsed_time(p1), dev, world)),
                    "unit": UNIT, "copies": "overlapped steps: uploads and read-backs on two copy streams "
                    "overlap the neighbouring steps' kernels (three buffer sets in turn, no L2 flush: the "
                    "other sets' steps read about 1.6x L2 between two uses of a set)"}
            prev = {"value": e2e["value"], "unit": UNIT, "copies": e2e["copies"]}
            if pipe["value"] > e2e["value"]:
                e2e["serial"] = prev
                e2e["value"], e2e["copies"] = pipe["value"], pipe["copies"]
            else:
                e2e["pipelined"] = pipe
            del sets, extra

    # roofline of the dominant kernel (largest share of the step); its duration comes from
    # the headline pass when that pass bracketed it
    avg = {n: statistics.mean(v) for n, v in per_stage.items()}
    dom = max(crit_names, key=lambda n: avg[n])
    dom_t = statistics.mean(dom_ms) if dom == dom_key and dom_ms else avg[dom]
    spec0 = runs[int(dom.split(":")[0])][0]
    bnd, _ = bound_of(dom, spec0, work, pk, args.attn_impl)
    b, f = work[dom]
    if bnd == "hbm":
        achieved = b / (dom_t / 1e3) / 1e9
        peak, unit = pk["hbm_gbs"], "GB/s"
    else:
        achieved = f / (dom_t / 1e3) / 1e12
        factor, mix = tensor_mix(dom, spec0, args.attn_impl)
        peak, unit = pk["bf16_tflops"] * factor, "TFLOP/s"
        pk_kind = f"{pk_kind} bf16 x {factor:.3g} ({mix}; nominal dtype ratio)"
    traffic = kernel_traffic(args.workload, dom.split(":")[1], args.attn_impl)
    stages = {}
    for n in stage_names:
        bb, ff = work[n]
        bn, t_roof = bound_of(n, runs[int(n.split(":")[0])][0], work, pk, args.attn_impl)
        stages[n] = {"ms": round(avg[n], 5), "share": round(avg[n] / sum(avg.values()), 4),
                     "bytes": int(bb), "flops": int(ff), "bound": bn,
                     "roofline_frac": round(t_roof * 1e3 / avg[n], 4) if avg[n] > 0 else None}

    status_ok = all(r.read_status() == 0 for _, _, r in runs)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3+bf16 KV, mxfp4 indexer, fp32 accumulate" if not runs[0][0].fp32 else "f32",
        "data": "synthetic",
        "config": {**workload_config(args.workload), "query_tokens_per_step_per_gpu": units,
                   "l2": "flushed between timed steps, outside the step events (512 MiB write, then a "
                         "256 MiB read so that evicted lines are clean)",
                   "launch": "eager" if graph is None else "cuda graph of the step",
                   "stage_times": "eager steps" if graph is None else
                   "third timed pass, every stage bracketed by graph event nodes",
                   "kernel_time": "eager steps" if graph is None else
                   "second timed pass, the dominant stage bracketed by graph event nodes",
                   "parallelism": f"replicas x{world} (independent batches)"},
        "roofline": {"bound": bnd, "kernel": dom.split(":")[1], "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak, "traffic": traffic, "peak_source": pk_kind,
                     "ms_per_launch": dom_t},
        "stages": stages,
        "gpu_launches": n_launch * args.steps,
        "clocks": clk.summary(),
        "e2e": e2e,
        "status_ok": status_ok,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_sample_s)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------------------------
# the oracle (CPU baseline / reference arm)
# ------------------------------------------------------------------------------------
def _one_thread():
    """Context that limits numpy's BLAS to one thread: the oracle is timed single-threaded
    on one host core."""
    from threadpoolctl import threadpool_limits
    return threadpool_limits(limits=1)


def _lc_libs_mapped():
    """Shared objects of this library mapped into the process (the oracle legs load none)."""
    try:
        with open("/proc/self/maps") as f:
            return sorted({ln.split()[-1] for ln in f if ln.rstrip().endswith("liblc.so")})
    except OSError:
        return []


def oracle_unit(name: str):
    """A callable that processes ONE query token of the workload with the oracle (host
    inputs drawn with the same generators), plus a description."""
    import numpy as np
    from long_context_sparse_softmax_b200 import workloads as wl
    from oracle import lc_oracle as O
    from oracle import pipeline as P
    spec = wl.WORKLOADS[name][0]
    if spec.is_decode:
        # one sequence of the batch: index over its whole visible cache, top-k, attention
        one = wl.shrink(spec, seq_lens=spec.seq_lens[:1])
        inp = wl.make_decode(one, "cpu")
        cache = inp["cache"]
        ent = O.rows_to_f64(one.kv_fmt, cache["x"].numpy(), cache.get("rope").numpy() if "rope" in cache else None)
        win = O.rows_to_f64(one.win_fmt, inp["win"].numpy())
        p = one.seq_lens[0] - 1
        qr = P.raw_rows(one.raw_fmt, inp["q_raw"].numpy())
        sink = inp["sink"].numpy().astype(np.float64)

        def unit():
            q, _, _ = P.stored(one.q_fmt, O.qk_prep(qr, np.array([p]), one.rope_off, one.d_r), one.d_n)
            if one.is_csa:
                if one.idx_fmt == O.IDX_MXFP4:
                    qI = O.mxfp4_to_f64(*O.f64_to_mxfp4(O.bf16_to_f64(inp["qI_raw"].numpy())))[0]
                else:
                    qI = P.indexer_f64(one.idx_fmt, {k: v.numpy() for k, v in inp["qI"].items()})[0]
                kI = P.indexer_f64(one.idx_fmt, {k: v.numpy() for k, v in inp["kI"].items()})
                idx, _, _ = P.select(qI, kI, inp["w"].numpy().astype(np.float64), p, one.m, one.W, one.k)
            else:
                idx = range(O.n_visible(p, one.m, one.W, ent.shape[0]))
            return O.sparse_attn_query(q[0], ent, idx, win, max(0, p - one.W + 1), p, one.W, sink, one.scale)
        return unit, f"{name}: one sequence (context {one.seq_lens[0]}) per unit, float64 oracle"
    # prefill: one query of the sequence (entries compressed once, outside the timing)
    small_n = 1
    inp = wl.make_prefill(spec, "cpu")
    x_bits = inp["x"].numpy()
    xfun = lambda r0, n: P.raw_rows(spec.raw_fmt, x_bits[r0:r0 + n])
    ent, _, _ = P.entries_from_tokens(xfun, inp["g"].numpy().astype(np.float64), spec.m, spec.rope_off, spec.d_r,
                                      spec.kv_fmt, spec.d_n)
    sink = inp["sink"].numpy().astype(np.float64)
    kI_all = None
    if spec.is_csa:
        if spec.idx_fmt == O.IDX_MXFP4:
            pooled = O.pool_index_keys(O.bf16_to_f64(inp["kI_raw"].numpy()), inp["g"].numpy().astype(np.float64), spec.m)
            kI_all = O.mxfp4_to_f64(*O.f64_to_mxfp4(pooled))
        else:
            kI_all = P.indexer_f64(spec.idx_fmt, {k: v.numpy() for k, v in inp["kI"].items()})
    rng = np.random.default_rng(0)
    qs = rng.integers(0, spec.n_q, 64)
    state = {"i": 0}

    def unit():
        i = int(qs[state["i"] % len(qs)])
        state["i"] += 1
        p = spec.q_first + i
        ts = list(O.window_positions(p, spec.W))
        raw = P.raw_rows(spec.raw_fmt, x_bits[ts])
        win, _, _ = P.stored(spec.win_fmt, O.qk_prep(raw, np.array(ts), spec.rope_off, spec.d_r), spec.d_n)
        qr = P.raw_rows(spec.raw_fmt, inp["q_raw"][i:i + 1].numpy())
        q, _, _ = P.stored(spec.q_fmt, O.qk_prep(qr, np.array([p]), spec.rope_off, spec.d_r), spec.d_n)
        if spec.is_csa:
            if spec.idx_fmt == O.IDX_MXFP4:
                qI = O.mxfp4_to_f64(*O.f64_to_mxfp4(O.bf16_to_f64(inp["qI_raw"][i:i + 1].numpy())))[0]
            else:
                qI = P.indexer_f64(spec.idx_fmt, {k: v[i:i + 1].numpy() for k, v in inp["qI"].items()})[0]
            idx, _, _ = P.select(qI, kI_all, inp["w"].numpy().astype(np.float64), p, spec.m, spec.W, spec.k)
        else:
            idx = range(O.n_visible(p, spec.m, spec.W, ent.shape[0]))
        return O.sparse_attn_query(q[0], ent, idx, win, ts[0], p, spec.W, sink, spec.scale)
    return unit, f"{name}: one query per unit (entries and indexer keys compressed once beforehand), float64 oracle"


def cpu_baseline(name: str, budget_s: float):
    unit, desc = oracle_unit(name)
    with _one_thread():
        unit()
        n, t0 = 0, time.perf_counter()
        while True:
            unit()
            n += 1
            el = time.perf_counter() - t0
            if el >= budget_s or n >= 10000:
                break
    return {"value": n / el, "unit": UNIT, "cores": 1, "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{desc}; {n} units in {el:.1f} s, one thread"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    unit, desc = oracle_unit(args.workload)
    t = []
    with _one_thread():
        for _ in range(args.warmup):
            unit()
        for _ in range(args.steps):
            t0 = time.perf_counter()
            unit()
            t.append(time.perf_counter() - t0)
    total = sum(t)
    value = args.steps / total
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**workload_config(args.workload), "sample": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "host_cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"{desc}; one unit per step, one thread"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "native_libs_loaded": _lc_libs_mapped(),
    }), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_lc(a)
