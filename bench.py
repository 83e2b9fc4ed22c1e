#!/usr/bin/env python
"""LSA hot-path benchmark on B200.

Headline: LSA decode tokens/s/layer at 128K context. Workload: batch 16, every
sequence at cached length 131072, 14 layers, each layer one index pass
(lightning indexer over all 131072 keys, top-2048 with 16 sink + 1024 local
forced) feeding two attention sub-blocks of sparse absorbed-latent MLA over
independent latent caches. One step = one decode token for every sequence
through all 14 layers. tokens/s/layer = batch * 14 / step time. Per step the
caches read are ~8.6 GB (> L2), so no L2 flush is needed between steps.

Also reported: prefill tok/s of one 16384-token causal sequence (same path in
prefill form), the roofline fraction of the dominant kernel, the fp64 CPU
oracle on a bounded sample, an end-to-end number through lsa_forward with
pinned host buffers and host<->device copies inside the timed region, and an
MTP draft round ("mtp": one index pass and top-k per layer shared by three
draft steps of sparse MLA over one latent cache; tokens = 3 per sequence per
layer per round), and the indexer's own projections with the key-cache append
("project": one decode token per sequence per layer, with its HBM roofline),
and the decode step with hierarchical indexing ("hier": per layer the newest
block's summary, a coarse pass over 64-key block summaries keeping the sink /
recent blocks and the 128 best others, the fine selection over their tokens,
then both MLA sub-blocks; also the selection alone against the flat index pass
and top-k), LoZA attention over the same decode workload ("loza": per layer both
sub-blocks over each row's sink, recent window and own chunk, no indexer; with
its HBM roofline), and the other workloads of the pages' configuration list as one
lsa_forward layer each ("configs": single-token decode latency at 8192 cached
keys with L2 flushed before every step, 64 sequences of 16K-32K cached keys,
4 sequences at 983040, and a 4096-token prefill chunk against 983040).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference]
Multi-GPU (torchrun): every rank runs its own batch (weak scaling, no
collective on the data path); rank 0 prints the aggregate.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import lsa_synth as S  # noqa: E402

METRIC = "LSA decode tokens/s/layer at 128K ctx"
DECODE = dict(batch=16, ctx=131072, layers=14, cli=2)
PREFILL = dict(seq=16384)
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# multi-process plumbing
# ---------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))


def reduce_max(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate(units_per_rank: float, seconds_per_rank: float, world: int, device=None):
    """Whole-job throughput: units of all ranks / the slowest rank's time."""
    t = reduce_max(seconds_per_rank, world, device)
    return units_per_rank * world / t, t


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.idx = device_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# the decode indexer's code: its kernel and its key-tile helpers
INDEX_DECODE_SOURCES = ("index_decode.cu", "index_tile.cuh")
INDEX_PREFILL_SOURCES = ("index_prefill.cu", "tc.cuh")


def source_sha(srcs) -> str:
    """sha256 over the kernel's source files (in order) under csrc/."""
    h = hashlib.sha256()
    for src in srcs:
        h.update(open(os.path.join(ROOT, "sparse_attention_03_b200", "csrc", src), "rb").read())
    return h.hexdigest()


def kernel_traffic(kernel: str, srcs):
    """dram bytes per launch from the committed ncu summary, if it was taken on these sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d:
        return None
    return d["bytes_per_launch"] if d.get("source_sha256") == source_sha(srcs) else None


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample (rank 0, N=1 only; also the reference arm)
# ---------------------------------------------------------------------------
class OracleSample:
    """Host inputs for a few decode rows of the 128K workload (drawn untimed)."""

    def __init__(self, n_rows: int, layer: int = 0):
        ctx = DECODE["ctx"]
        self.rows = []
        f = S.bf16_bits_to_f64
        for b in range(n_rows):
            q = f(S.normal_bf16(0, S.tid(layer, S.Q_IDX), b * 4096, 4096)).reshape(32, 128)
            w = S.normal_f32(0, S.tid(layer, S.W), b * 32, 32, S.W_SIGMA).astype(np.float64)
            k = f(S.rms_rows_bf16(0, S.tid(layer, S.K_IDX), b * ctx, ctx, 128))
            qa = [f(S.normal_bf16(0, S.tid(layer, S.q_abs_kind(z)), b * 32 * 576, 32 * 576)).reshape(32, 576)
                  for z in range(2)]
            # Drawing 2 x 75M latent values on the host takes far longer than the
            # oracle itself; draw only the rows this query selects (found by one
            # untimed oracle pass) and gather from that table in the timed unit.
            from oracle import lsa_ref as R
            p = ctx - 1
            sel0, _ = R.select_topk(R.mask_and_force(R.score_row(q, w, k), p, ctx, R.PAGES), p, R.PAGES)
            lat = [S.normal_bf16_rows(0, S.tid(layer, S.lat_kind(z)), b * ctx + sel0, 576) for z in range(2)]
            self.rows.append((q, w, k, qa, sel0, lat))

    def unit(self, i):
        """One decode token of one sequence through one layer, as the oracle computes it
        (inputs already drawn; selected latent rows are gathered and widened to fp64)."""
        from oracle import lsa_ref as R
        q, w, k, qa, sel0, lat = self.rows[i % len(self.rows)]
        p = DECODE["ctx"] - 1
        s = R.mask_and_force(R.score_row(q, w, k), p, DECODE["ctx"], R.PAGES)
        sel, _ = R.select_topk(s, p, R.PAGES)
        at = np.searchsorted(sel0, sel)
        for z in range(2):
            R.mla(qa[z], S.bf16_bits_to_f64(lat[z][at]), R.PAGES)


def oracle_rate(sample: OracleSample, budget_s: float):
    n, t0 = 0, time.perf_counter()
    while True:
        sample.unit(n)
        n += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return n, time.perf_counter() - t0


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(budget_s: float = 12.0):
    sample = OracleSample(2)
    sample.unit(0)  # warm BLAS
    n, t = oracle_rate(sample, budget_s)
    return {"value": n / t, "unit": "tokens/s/layer", "cores": host_cores(), "kind": "oracle",
            "sample": f"{n} decode tokens (one sequence through one layer each: indexer over 131072 keys, "
                      f"top-2048, 2 sub-blocks of sparse MLA) of the 128K workload, fp64 numpy, {t:.1f} s"}


def reference_arm(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    sample = OracleSample(2)
    sample.unit(0)
    for _ in range(args.warmup):
        sample.unit(1)
    per_step = 4
    t0 = time.perf_counter()
    for s in range(args.steps):
        for u in range(per_step):
            sample.unit(s * per_step + u)
    t = time.perf_counter() - t0
    units = args.steps * per_step
    v = units / t
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s/layer", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": "decode_b16_ctx131072_14layers_cli2",
                                            "sample": f"{per_step} decode tokens per step"},
            "cpu_baseline": {"value": v, "unit": "tokens/s/layer", "cores": host_cores(), "kind": "oracle",
                             "sample": f"{units} decode tokens of the 128K workload, fp64 numpy"},
            "e2e": {"value": v, "unit": "tokens/s/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def build_decode(device):
    import torch
    from sparse_attention_03_b200 import lsa
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    B, ctx, nl = DECODE["batch"], DECODE["ctx"], DECODE["layers"]
    lengths = np.full(B, ctx, dtype=np.int64)
    layers = [DeviceWorkload(0, l, lengths, device=device) for l in range(nl)]
    # per-step inputs and outputs of all layers in single buffers (one copy each way)
    q_idx = torch.stack([l.q_idx for l in layers]).contiguous()
    w = torch.stack([l.w for l in layers]).contiguous()
    q_abs = torch.stack([torch.stack(l.q_abs) for l in layers]).contiguous()
    for i, l in enumerate(layers):
        l.q_idx, l.w, l.q_abs = q_idx[i], w[i], [q_abs[i, 0], q_abs[i, 1]]
    out = torch.empty((nl, 2, B, 32, 512), dtype=torch.bfloat16, device=device)
    lse = torch.empty((nl, 2, B, 32), dtype=torch.float32, device=device)
    cfg = lsa.LsaConfig()
    ws = lsa.workspace(cfg, lsa.OP_FORWARD_DECODE, B, B, ctx, device=device)
    scores = torch.empty((B, ctx), dtype=torch.float32, device=device)
    idx = torch.empty((B, 2048), dtype=torch.int32, device=device)
    cnt = torch.empty((B,), dtype=torch.int32, device=device)
    tk_ws = lsa.workspace(cfg, lsa.OP_TOPK, B, B, ctx, device=device)
    mla_ws = lsa.workspace(cfg, lsa.OP_MLA_DECODE_LAYER, B, B, ctx, device=device)
    mtp_ws = lsa.workspace(cfg, lsa.OP_MTP_DECODE, B, B, ctx, device=device)
    hist = lsa.topk_hist_buffer(B, device=device)
    D = dict(layers=layers, q_idx=q_idx, w=w, q_abs=q_abs, out=out, lse=lse, cfg=cfg, ws=ws, scores=scores,
             idx=idx, cnt=cnt, tk_ws=tk_ws, mla_ws=mla_ws, mtp_ws=mtp_ws, ctx=ctx, hist=hist)
    # Marshal every call once: the timed loops only cross the C-ABI.
    D["calls"] = []
    D["two_launch"] = []
    D["fwd"] = []
    for i, l in enumerate(layers):
        D["calls"].append((
            lsa.index_scores(cfg, l.seq_of_row, l.pos, l.q_idx, l.w, l.k_idx, l.k_off, ctx, scores, bind=True,
                             topk_hist=hist),
            lsa.topk(cfg, l.pos, ctx, scores, idx, cnt, tk_ws, bind=True, topk_hist=hist),
            lsa.sparse_mla_decode_layer(cfg, l.q_abs, l.latent, l.k_off, idx, cnt, ctx, [out[i, 0], out[i, 1]],
                                        [lse[i, 0], lse[i, 1]], mla_ws, bind=True)))
        # the same sub-blocks as two launches (a model whose second sub-block's
        # query waits for the first one's output)
        D["two_launch"].append([lsa.sparse_mla_decode(cfg, l.q_abs[z], l.latent[z], l.k_off, idx, cnt, ctx,
                                                      out[i, z], lse[i, z], mla_ws, bind=True, lists_from_topk=True)
                                for z in range(2)])
        D["fwd"].append(lsa.forward(cfg, 0, l.seq_of_row, l.pos, ctx, l.q_idx, l.w, l.k_idx, l.k_off, l.q_abs,
                                    l.latent, [out[i, 0], out[i, 1]], [lse[i, 0], lse[i, 1]], ws, bind=True))
    # MTP draft round: the index pass and top-k once, for the first draft step's
    # query at position ctx - 3; the three draft steps (queries at ctx - 3,
    # ctx - 2, ctx - 1, each also seeing the later keys up to its own) in one
    # launch over one latent cache
    q3 = torch.empty((nl, B, 32, 576), dtype=torch.bfloat16, device=device)
    for i in range(nl):
        lsa.synth_normal_bf16(q3[i], 0, 16 * (100 + i) + 3)
    out3 = [torch.empty((B, 32, 512), dtype=torch.bfloat16, device=device) for _ in range(3)]
    lse3 = [torch.empty((B, 32), dtype=torch.float32, device=device) for _ in range(3)]
    pos3 = torch.full((B,), ctx - 3, dtype=torch.int32, device=device)
    D["mtp"] = []
    for i, l in enumerate(layers):
        D["mtp"].append((
            lsa.index_scores(cfg, l.seq_of_row, pos3, l.q_idx, l.w, l.k_idx, l.k_off, ctx, scores, bind=True,
                             topk_hist=hist),
            lsa.topk(cfg, pos3, ctx, scores, idx, cnt, tk_ws, bind=True, topk_hist=hist),
            lsa.mtp_mla_decode(cfg, pos3, [l.q_abs[0], l.q_abs[1], q3[i]], l.latent[0], l.k_off, idx, cnt, ctx,
                               out3, lse3, mtp_ws, bind=True)))
    D["mtp_keep"] = (q3, out3, lse3, pos3)
    return D


def build_project(D, device):
    """Per layer: the indexer's projection weights (wq_b, wk, weights_proj, key-norm
    weight) and one decode token's q-LoRA vector and hidden state per sequence."""
    import torch
    from sparse_attention_03_b200 import lsa
    import lsa_synth as S
    B, nl = DECODE["batch"], DECODE["layers"]
    ql, hd = 1536, 3072
    P = []
    for i, l in enumerate(D["layers"]):
        def draw(shape, kind, sigma=1.0):
            t = torch.empty(shape, dtype=torch.bfloat16, device=device)
            lsa.synth_normal_bf16(t, 0, S.tid(200 + i, kind), sigma=sigma)
            return t
        wq_b, wk, wp = draw((4096, ql), S.WQ_B, ql ** -0.5), draw((128, hd), S.WK, hd ** -0.5), draw((32, hd), S.WPROJ, hd ** -0.5)
        g = (1.0 + 0.1 * draw((128,), S.KNORM).float()).to(torch.bfloat16)
        c_q, h = draw((B, ql), S.C_Q), draw((B, hd), S.HIDDEN)
        q_out = torch.empty((B, 32, 128), dtype=torch.bfloat16, device=device)
        w_out = torch.empty((B, 32), dtype=torch.float32, device=device)
        ws = lsa.workspace(D["cfg"], lsa.OP_INDEX_PROJECT, B, B, D["ctx"], device=device)
        P.append(dict(keep=(wq_b, wk, wp, g, c_q, h, q_out, w_out, ws),
                      call=lsa.index_project(D["cfg"], l.seq_of_row, l.pos, l.k_off, D["ctx"], c_q, h, wq_b, wk, wp,
                                             g, q_out, w_out, l.k_idx, ws, bind=True)))
    D["project"] = P
    wbytes = (4096 * ql + 128 * hd + 32 * hd + 128) * 2
    io = B * ((ql + hd) * 2 + 32 * 128 * 2 + 32 * 4 + 128 * 2)
    D["project_bytes"] = wbytes + io


def build_hier(D, device, block=64, n_blocks=128):
    """Per layer: block summaries of the index-key cache (built once, untimed), the
    per-step update of each sequence's newest block, and the two-stage selection
    bound into the decode step's idx / count buffers."""
    import torch
    from sparse_attention_03_b200 import lsa
    B, ctx, cfg = DECODE["batch"], D["ctx"], D["cfg"]
    blk_off_h = lsa.block_offsets([ctx] * B, block)
    blk_off = torch.tensor(blk_off_h, dtype=torch.int64, device=device)
    nb = ctx // block if ctx % block == 0 else ctx // block + 1
    all_seq = torch.arange(B, dtype=torch.int32, device=device).repeat_interleave(nb)
    all_blk = torch.arange(nb, dtype=torch.int32, device=device).repeat(B)
    new_seq = torch.arange(B, dtype=torch.int32, device=device)
    new_blk = torch.full((B,), (ctx - 1) // block, dtype=torch.int32, device=device)
    ws = lsa.hier_workspace(cfg, B, ctx, block, n_blocks, device=device)
    H = []
    for l in D["layers"]:
        k_blk = torch.empty((blk_off_h[-1], 128), dtype=torch.bfloat16, device=device)
        lsa.block_summaries(cfg, all_seq, all_blk, l.k_idx, l.k_off, blk_off, k_blk, block)
        H.append(dict(k_blk=k_blk,
                      update=lsa.block_summaries(cfg, new_seq, new_blk, l.k_idx, l.k_off, blk_off, k_blk, block,
                                                 bind=True),
                      select=lsa.hier_select(cfg, l.seq_of_row, l.pos, l.q_idx, l.w, l.k_idx, l.k_off, k_blk,
                                             blk_off, ctx, D["idx"], D["cnt"], ws, block, n_blocks, bind=True)))
    D["hier"] = H
    D["hier_keep"] = (blk_off, all_seq, all_blk, new_seq, new_blk, ws)
    D["hier_cfg"] = {"block": block, "n_blocks": n_blocks}


LOZA_PATTERN = (16, 1024, 4096)  # sink, recent, chunk


def build_loza(D, device):
    """Per layer: both sub-blocks' LoZA attention (sink, recent window, own chunk)
    over the same caches and queries as the decode step; no indexer."""
    from sparse_attention_03_b200 import lsa
    B, ctx, cfg = DECODE["batch"], D["ctx"], D["cfg"]
    ws = lsa.workspace(cfg, lsa.OP_MLA_DECODE, B, B, ctx, device=device)
    D["loza_ws"] = ws
    D["loza"] = [[lsa.loza_mla(cfg, LOZA_PATTERN, 0, l.seq_of_row, l.pos, l.k_off, ctx, l.q_abs[z], l.latent[z],
                               D["out"][i, z], D["lse"][i, z], ws, bind=True) for z in range(2)]
                 for i, l in enumerate(D["layers"])]
    p = ctx - 1
    s_end = min(LOZA_PATTERN[0], ctx)
    w0 = max(min(p - LOZA_PATTERN[1] + 1, p // LOZA_PATTERN[2] * LOZA_PATTERN[2]), s_end)
    D["loza_keys"] = s_end + ctx - w0


def loza_step(D):
    for calls in D["loza"]:
        for call in calls:
            call()


def hier_step(D, select_only=False):
    """One decode step with hierarchical selection: per layer the newest block's
    summary, the two-stage selection, then both MLA sub-blocks on it."""
    for h, (_, _, mla_call) in zip(D["hier"], D["calls"]):
        h["update"]()
        h["select"]()
        if not select_only:
            mla_call()


def flat_select_step(D):
    for idx_call, topk_call, _ in D["calls"]:
        idx_call()
        topk_call()


def project_step(D):
    for p in D["project"]:
        p["call"]()


def mtp_round(D):
    """One MTP draft round through every layer: the index pass and top-k once,
    then the three draft steps of sparse MLA over that one selection (one launch)."""
    for idx_call, topk_call, mtp_call in D["mtp"]:
        idx_call()
        topk_call()
        mtp_call()


def decode_step(D, ev=None, mla_ev=None):
    """One decode step through every layer via the C-ABI entry points (index pass,
    top-k, both sub-blocks of sparse MLA in one launch). If `ev` (`mla_ev`) is
    given, records events on the launching stream around each indexer (attention)
    launch."""
    for i, (idx_call, topk_call, mla_call) in enumerate(D["calls"]):
        if ev is not None:
            ev[i][0].record()
        idx_call()
        if ev is not None:
            ev[i][1].record()
        topk_call()
        if mla_ev is not None:
            mla_ev[i][0].record()
        mla_call()
        if mla_ev is not None:
            mla_ev[i][1].record()


def decode_step_two_launch(D):
    """The same step with the two sub-blocks' attention as two launches."""
    for (idx_call, topk_call, _), mla_calls in zip(D["calls"], D["two_launch"]):
        idx_call()
        topk_call()
        mla_calls[0]()
        mla_calls[1]()


def build_e2e_sets(D, device):
    """Two sets of per-step device buffers (queries in, attention out) with
    lsa_forward bound to each, so that one step's host copies travel while the
    other set computes."""
    import torch
    from sparse_attention_03_b200 import lsa
    sets = [dict(q_idx=D["q_idx"], w=D["w"], q_abs=D["q_abs"], out=D["out"], lse=D["lse"], fwd=D["fwd"])]
    qi, w, qa = D["q_idx"].clone(), D["w"].clone(), D["q_abs"].clone()
    out, lse = torch.empty_like(D["out"]), torch.empty_like(D["lse"])
    fwd = [lsa.forward(D["cfg"], 0, l.seq_of_row, l.pos, D["ctx"], qi[i], w[i], l.k_idx, l.k_off, [qa[i, 0], qa[i, 1]],
                       l.latent, [out[i, 0], out[i, 1]], [lse[i, 0], lse[i, 1]], D["ws"], bind=True)
           for i, l in enumerate(D["layers"])]
    sets.append(dict(q_idx=qi, w=w, q_abs=qa, out=out, lse=lse, fwd=fwd))
    return sets


def decode_forward_e2e(sets, s, h_in, h_out, pipe, last=False):
    """Step s through lsa_forward (every layer), its inputs copied from pinned
    host memory and its outputs (attention output and lse of every layer)
    copied back. Steps alternate between two sets of device buffers: step s's
    input copy (one stream) runs while step s-1 computes, and its output copy
    (another stream) while step s+1 computes; the compute stream waits for
    those copies once per step, so the layers' kernels stay back to back. With
    last=True the compute stream also waits for this step's output copy, which
    ends the timed region after every copy of every step."""
    import torch
    comp, h2d, d2h, evs = pipe
    X, ev = sets[s % 2], evs[s % 2]
    with torch.cuda.stream(h2d):
        h2d.wait_event(ev["done"])              # this set's previous step has read its inputs
        X["q_idx"].copy_(h_in[0], non_blocking=True)
        X["w"].copy_(h_in[1], non_blocking=True)
        X["q_abs"].copy_(h_in[2], non_blocking=True)
        ev["in"].record(h2d)
    comp.wait_event(ev["in"])
    comp.wait_event(ev["out"])                  # this set's previous outputs have been copied out
    for call in X["fwd"]:
        call()
    ev["done"].record(comp)
    with torch.cuda.stream(d2h):
        d2h.wait_event(ev["done"])
        h_out[0].copy_(X["out"], non_blocking=True)
        h_out[1].copy_(X["lse"], non_blocking=True)
        ev["out"].record(d2h)
    if last:
        comp.wait_stream(d2h)
        comp.wait_stream(h2d)


def time_region(fn, steps, world, device):
    import torch
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for s in range(steps):
        fn(s)
    b.record()
    torch.cuda.synchronize()
    barrier(world)
    return a.elapsed_time(b) / 1e3


def run_prefill(device, steps, warmup):
    import torch
    from sparse_attention_03_b200 import lsa
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    n = PREFILL["seq"]
    wl = DeviceWorkload(0, 100, [n], n_rows=n, q_start=0, device=device)
    cfg = lsa.LsaConfig()
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device=device) for _ in range(2)]
    lses = [torch.empty((n, 32), device=device) for _ in range(2)]
    ws = lsa.workspace(cfg, lsa.OP_FORWARD_PREFILL, n, 1, n, device=device)
    scores = torch.empty((n, n), device=device)
    idx = torch.empty((n, 2048), dtype=torch.int32, device=device)
    cnt = torch.empty((n,), dtype=torch.int32, device=device)
    tk_ws = lsa.workspace(cfg, lsa.OP_TOPK, n, 1, n, device=device)
    mla_ws = lsa.workspace(cfg, lsa.OP_MLA_PREFILL, n, 1, n, device=device)
    ev = []
    idx_call = lsa.index_scores(cfg, None, wl.pos, wl.q_idx, wl.w, wl.k_idx, None, n, scores, bind=True)
    topk_call = lsa.topk(cfg, wl.pos, n, scores, idx, cnt, tk_ws, bind=True)
    mla_calls = [lsa.sparse_mla_prefill(cfg, wl.pos, wl.q_abs[z], wl.latent[z], idx, cnt, outs[z], lses[z],
                                        mla_ws, bind=True) for z in range(2)]

    def step(record):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        idx_call()
        e1.record()
        if record:
            ev.append((e0, e1))
        topk_call()
        mla_calls[0]()
        mla_calls[1]()

    for _ in range(warmup):
        step(False)
    t = time_region(lambda s: step(True), steps, 1, device)
    idx_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = 2.0 * 32 * 128 * (n * (n + 1) / 2)  # visible (row, key) pairs
    pk, src = peaks()
    peak = pk["bf16_tflops"]  # the burst figure: a ~1 ms kernel, not a seconds-long loop
    achieved = flops / (idx_ms / 1e3) / 1e12
    del wl, scores
    torch.cuda.empty_cache()
    return {"value": n * steps / t, "unit": "tok/s", "ms_per_step": 1e3 * t / steps,
            "config": {"workload": "prefill_causal_16384", "seq_len": n},
            "roofline": {"kernel": "index_prefill_kernel", "bound": "tensor",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{src} bf16_tflops (burst)",
                         "traffic": kernel_traffic("index_prefill_kernel", INDEX_PREFILL_SOURCES)}}


def _forward_case(device, lengths, n_rows=None, q_start=None, layer=300):
    """One layer's lsa_forward call (cli 2) on device-drawn inputs, bound once."""
    import torch
    from sparse_attention_03_b200 import lsa
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    cfg = lsa.LsaConfig()
    wl = DeviceWorkload(0, layer, lengths, n_rows=n_rows, q_start=q_start, device=device)
    n, max_len = wl.n_rows, wl.max_len
    mode = 0 if n_rows is None else 1
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device=device) for _ in range(2)]
    lses = [torch.empty((n, 32), device=device) for _ in range(2)]
    n_seq = len(lengths) if mode == 0 else 1
    ws = lsa.workspace(cfg, lsa.OP_FORWARD_DECODE if mode == 0 else lsa.OP_FORWARD_PREFILL, n, n_seq, max_len,
                       device=device)
    call = lsa.forward(cfg, mode, wl.seq_of_row, wl.pos, max_len, wl.q_idx, wl.w, wl.k_idx, wl.k_off, wl.q_abs,
                       wl.latent, outs, lses, ws, bind=True)
    return call, (wl, outs, lses, ws)


def run_configs(device, steps):
    """The other workloads of the pages' configuration list, one lsa_forward layer
    (one index pass, top-k, two sub-blocks) per step: single-token latency at
    8192 cached keys (caches fit in L2, so L2 is flushed before every step and
    each step is event-timed alone; and, as inside a model's forward, 14 such
    layers back to back, whose caches together exceed L2), the 64-sequence
    varlen decode, and the
    long-context pair (4 sequences at 983040 cached keys; a 4096-token prefill
    chunk against the 983040-token cache)."""
    import torch
    from sparse_attention_03_b200 import lsa
    res = {}

    # decode, batch 1, 8192 cached keys: latency with a cold L2
    call, keep = _forward_case(device, [8192])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    lat = []
    for i in range(steps + 3):
        flush.fill_(i & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        torch.cuda.synchronize()
        if i >= 3:
            lat.append(a.elapsed_time(b))
    res["decode_b1_ctx8192"] = {"value": 1e3 / statistics.median(lat), "unit": "tokens/s/layer",
                                "us_per_layer": 1e3 * statistics.median(lat),
                                "l2": "flushed (256 MB write) before every step; median of per-step events"}
    del call, keep, flush

    def timed(call, units, n_steps):
        for _ in range(3):
            call()
        t = time_region(lambda s: call(), n_steps, 1, device)
        return units * n_steps / t, 1e3 * t / n_steps

    # the same single-token layer, 14 layers (each with its own caches) per step
    cases = [_forward_case(device, [8192], layer=300 + i) for i in range(14)]
    v, ms = timed(lambda: [c() for c, _ in cases], 14, steps)
    res["decode_b1_ctx8192_14layers"] = {"value": v, "unit": "tokens/s/layer", "us_per_layer": 1e3 * ms / 14,
                                         "l2": "14 layers' caches (0.30 GB) per step, no flush"}
    del cases
    torch.cuda.empty_cache()

    # decode, batch 64, cached lengths uniform in [16384, 32768]
    lengths = S.decode_lengths(0, 64, 16384, 32768)
    call, keep = _forward_case(device, lengths)
    v, ms = timed(call, 64, steps)
    res["decode_b64_ctx16k_32k"] = {"value": v, "unit": "tokens/s/layer", "ms_per_layer": ms,
                                    "cached_keys": int(lengths.sum()),
                                    "l2": f"{int(lengths.sum()) * 2560 / 1e9:.1f} GB of caches per step, no flush"}
    del call, keep
    torch.cuda.empty_cache()

    # decode, batch 4, 983040 cached keys
    call, keep = _forward_case(device, [983040] * 4)
    v, ms = timed(call, 4, steps)
    res["decode_b4_ctx983040"] = {"value": v, "unit": "tokens/s/layer", "ms_per_layer": ms,
                                  "l2": "10.1 GB of caches per step, no flush"}
    del call, keep
    torch.cuda.empty_cache()

    # prefill chunk of 4096 tokens at positions 983040 .. 987135
    n, q0 = 4096, 983040
    call, keep = _forward_case(device, [q0 + n], n_rows=n, q_start=q0)
    v, ms = timed(call, n, max(3, steps // 4))
    flops = 2.0 * 32 * 128 * (n * q0 + n * (n + 1) / 2)  # visible (row, key) pairs of the indexer
    res["prefill_chunk4096_ctx983040"] = {"value": v, "unit": "tok/s", "ms_per_chunk": ms,
                                          "indexer_tflop": flops / 1e12,
                                          "l2": "16 GB score matrix and 2.5 GB of caches per step, no flush"}
    del call, keep
    torch.cuda.empty_cache()
    return res


def gpu_arm(args):
    import torch
    from sparse_attention_03_b200 import lsa
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init(world, "nccl")
    lsa.load()
    D = build_decode(device)
    nl, B = DECODE["layers"], DECODE["batch"]

    def events():
        return [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(nl)]

    for _ in range(args.warmup):
        decode_step(D)
    torch.cuda.synchronize()
    assert lsa.device_error() == 0

    # kernel-level timed region (inputs resident in HBM); events on the launching
    # (current) stream bracket the indexer launches of the last timed step only:
    # an event between two kernels keeps the second from launching while the
    # first finishes, so instrumenting every step would slow the step it measures.
    ev_last = events()
    with ClockSampler(local) as clk:
        l0 = lsa.launch_count()
        barrier(world)
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for s in range(args.steps):
            decode_step(D, ev_last if s == args.steps - 1 else None)
        t1.record()
        torch.cuda.synchronize()
        barrier(world)
        launches = lsa.launch_count() - l0
    t = t0.elapsed_time(t1) / 1e3
    idx_ms = [a.elapsed_time(b) for a, b in ev_last]
    units = B * nl * args.steps
    value, tmax = aggregate(units, t, world, device)

    # roofline of the dominant kernel (the indexer: 256 B of k_idx + 4 B of score per key)
    keys = B * DECODE["ctx"]
    alg_bytes = keys * (256 + 4) + B * (32 * 128 * 2 + 32 * 4)
    pk, psrc = peaks()
    peak = pk["hbm_gbs"]
    achieved = alg_bytes / (statistics.mean(idx_ms) / 1e3) / 1e9

    # roofline of the attention kernel (both sub-blocks in one launch): events
    # around each MLA launch in separate untimed steps (an event between two
    # kernels stops the second from starting early, so the timed steps carry none)
    mla_ev = events()
    for _ in range(3):
        decode_step(D, mla_ev=mla_ev)
    torch.cuda.synchronize()
    mla_ms = statistics.mean(a.elapsed_time(b) for a, b in mla_ev)
    mla_bytes = B * 2 * (2048 * 1152 + 32 * 576 * 2 + 32 * 512 * 2 + 32 * 4)
    mla_achieved = mla_bytes / (mla_ms / 1e3) / 1e9

    # the same step with the sub-blocks' attention as two launches
    for _ in range(3):
        decode_step_two_launch(D)
    t2 = time_region(lambda s: decode_step_two_launch(D), args.steps, world, device)
    two_value, _ = aggregate(units, t2, world, device)

    # end-to-end through lsa_forward with pinned host buffers
    h_in = [D["q_idx"].cpu().pin_memory(), D["w"].cpu().pin_memory(), D["q_abs"].cpu().pin_memory()]
    h_out = [torch.empty(D["out"].shape, dtype=D["out"].dtype).pin_memory(),
             torch.empty(D["lse"].shape, dtype=D["lse"].dtype).pin_memory()]
    sets = build_e2e_sets(D, device)
    pipe = (torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream(),
            [dict(**{k: torch.cuda.Event() for k in ("in", "done", "out")}) for _ in range(2)])
    n_warm = max(3, args.warmup // 2)
    for w_ in range(n_warm):
        decode_forward_e2e(sets, w_, h_in, h_out, pipe, last=w_ == n_warm - 1)
    torch.cuda.synchronize()
    e2e_steps = max(5, args.steps // 2)
    te = time_region(lambda s: decode_forward_e2e(sets, s, h_in, h_out, pipe, last=s == e2e_steps - 1), e2e_steps,
                     world, device)
    e2e_value, _ = aggregate(B * nl * e2e_steps, te, world, device)
    h2d = sum(x.numel() * x.element_size() for x in h_in)
    d2h = sum(x.numel() * x.element_size() for x in h_out)

    # the indexer's own projections and key append for one decode token per sequence
    # (runs after the timed decode step: it rewrites the newest key row of each cache)
    build_project(D, device)
    D_bytes = D["project_bytes"]
    for _ in range(3):
        project_step(D)
    pj_steps = max(5, args.steps // 2)
    tp = time_region(lambda s: project_step(D), pj_steps, world, device)
    pj_value, _ = aggregate(B * nl * pj_steps, tp, world, device)
    pj_layer_s = tp / (pj_steps * nl)

    # MTP draft rounds (three draft tokens per sequence and layer per round)
    for _ in range(3):
        mtp_round(D)
    mtp_steps = max(5, args.steps // 2)
    tm = time_region(lambda s: mtp_round(D), mtp_steps, world, device)
    mtp_value, _ = aggregate(3 * B * nl * mtp_steps, tm, world, device)
    assert lsa.device_error() == 0

    # hierarchical indexing: the same decode step with the two-stage selection,
    # and the selection alone against the flat index pass + top-k
    build_hier(D, device)
    for _ in range(3):
        hier_step(D)
    h_steps = max(5, args.steps // 2)
    th = time_region(lambda s: hier_step(D), h_steps, world, device)
    hier_value, _ = aggregate(B * nl * h_steps, th, world, device)
    ths = time_region(lambda s: hier_step(D, select_only=True), h_steps, world, device)
    tfs = time_region(lambda s: flat_select_step(D), h_steps, world, device)
    assert lsa.device_error() == 0

    # LoZA attention: the same two sub-blocks per layer over the static pattern
    build_loza(D, device)
    for _ in range(3):
        loza_step(D)
    lz_steps = max(5, args.steps // 2)
    tl = time_region(lambda s: loza_step(D), lz_steps, world, device)
    loza_value, _ = aggregate(B * nl * lz_steps, tl, world, device)
    loza_keys = D["loza_keys"]
    assert lsa.device_error() == 0

    D_hier_cfg = D["hier_cfg"]
    del D
    torch.cuda.empty_cache()
    prefill = None
    if not args.no_prefill:
        prefill = run_prefill(device, max(3, args.steps // 20), 3)
    configs = None
    if not args.no_configs:
        configs = run_configs(device, max(5, args.steps // 10))

    clocks = clk.summary()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s/layer", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tmax / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "decode_b16_ctx131072_14layers_cli2", "batch": B, "ctx": DECODE["ctx"],
                   "layers": nl, "cli_factor": 2, "index_topk": 2048, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (8.6 GB of caches read per step), no flush"},
        "roofline": {"kernel": "index_decode_kernel", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_source": f"{psrc} hbm_gbs",
                     "traffic": kernel_traffic("index_decode_kernel", INDEX_DECODE_SOURCES),
                     "alg_bytes_per_launch": alg_bytes, "avg_launch_ms": statistics.mean(idx_ms)},
        "e2e": {"value": e2e_value, "unit": "tokens/s/layer", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline_attention": {"kernel": "mla_kernel", "bound": "hbm", "achieved": mla_achieved, "peak": peak,
                               "unit": "GB/s", "frac": mla_achieved / peak, "peak_source": f"{psrc} hbm_gbs",
                               "alg_bytes_per_launch": mla_bytes, "avg_launch_ms": mla_ms,
                               "timing": "events around each launch in 3 untimed steps"},
        "gpu_launches": launches,
        "two_launch": {"value": two_value, "unit": "tokens/s/layer", "ms_per_step": 1e3 * t2 / args.steps,
                       "note": "both sub-blocks' attention as two launches (second query after the first output)"},
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
    }
    line["project"] = {"value": pj_value, "unit": "tokens/s/layer", "us_per_layer": 1e6 * pj_layer_s,
                       "config": {"workload": "index_project_b16_qlora1536_hidden3072_14layers"},
                       "roofline": {"bound": "hbm", "achieved": D_bytes / pj_layer_s / 1e9, "peak": peak,
                                    "unit": "GB/s", "frac": D_bytes / pj_layer_s / 1e9 / peak,
                                    "peak_source": f"{psrc} hbm_gbs"}}
    line["mtp"] = {"value": mtp_value, "unit": "tokens/s/layer", "ms_per_round": 1e3 * tm / mtp_steps,
                   "config": {"workload": "mtp_draft_round_b16_ctx131072_14layers", "draft_steps": 3,
                              "index_passes_per_round": 1}}
    hc = D_hier_cfg
    line["hier"] = {"value": hier_value, "unit": "tokens/s/layer", "ms_per_step": 1e3 * th / h_steps,
                    "select_us_per_layer": 1e6 * ths / (h_steps * nl),
                    "flat_select_us_per_layer": 1e6 * tfs / (h_steps * nl),
                    "config": {"workload": f"hier_decode_b16_ctx131072_14layers_block{hc['block']}"
                                           f"_keep{hc['n_blocks']}", **hc}}
    lz_bytes = B * 2 * loza_keys * 1152 + B * 2 * (32 * 576 * 2 + 32 * 512 * 2)  # per layer: rows read, q in, out
    lz_layer_s = tl / (lz_steps * nl)
    line["loza"] = {"value": loza_value, "unit": "tokens/s/layer", "ms_per_step": 1e3 * tl / lz_steps,
                    "config": {"workload": "loza_decode_b16_ctx131072_14layers_cli2",
                               "pattern": dict(zip(("sink", "recent", "chunk"), LOZA_PATTERN)),
                               "keys_per_row": loza_keys},
                    "roofline": {"bound": "hbm", "achieved": lz_bytes / lz_layer_s / 1e9, "peak": peak,
                                 "unit": "GB/s", "frac": lz_bytes / lz_layer_s / 1e9 / peak,
                                 "peak_source": f"{psrc} hbm_gbs"}}
    if prefill:
        line["prefill"] = prefill
    if configs:
        line["configs"] = configs
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lsa", "reference"], default="lsa")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' lines")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        reference_arm(args)
        return
    gpu_arm(args)
    rank, world, _ = dist_env()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
