"""Small single-kernel cases for profiling one kernel of the path under ncu.

    python -m sparse_attention_03_b200.profile_cases CASE [--reps N]

Each case draws its inputs on the device (a few GB at most, inputs larger than
L2 where the kernel streams from HBM), runs one entry point --reps times on the
current stream, checks the device error flags and exits. Cases:

  index_decode   lsa_index_scores with the top-k histogram, 16 rows x 131072 keys (one 128K decode layer)
  index_prefill  lsa_index_scores, 16384 causal rows over 16384 keys
  topk_decode    lsa_topk on 16 rows x 131072 scores, with the indexer's histogram
  topk_rows      lsa_topk on 512 rows x 500000 random scores (the one-CTA-per-row kernel, long rows)
  mla_decode     lsa_sparse_mla_decode, 16 rows x 2048 selected keys of 131072
  mla_prefill    lsa_sparse_mla_prefill, 4096 rows x 2048 selected keys of 16384
  mla_layer      lsa_sparse_mla_decode_layer (both sub-blocks in one launch) on the top-k's lists,
                 16 rows x 131072 keys
  decode_8k      lsa_forward (cli 2), 1 row x 8192 keys (single-token decode latency)
  decode_1m      lsa_forward (cli 2), 4 rows x 983040 keys (one long-context decode layer)
  chunk_1m       lsa_forward (cli 2), a 4096-row prefill chunk at positions 983040.. (16 GB of scores)
  prefill_16k    one prefill step of 16384 causal rows: lsa_index_scores, lsa_topk, then
                 lsa_sparse_mla_prefill for two sub-blocks
  hier_decode    lsa_block_summaries of each row's newest block + lsa_hier_select (64-key blocks,
                 128 kept), 16 rows x 131072 keys
"""
from __future__ import annotations

import argparse
import sys

import numpy as np
import torch


from . import lsa
from .device_inputs import DeviceWorkload


def _decode_layer(draw_latent):
    lengths = np.full(16, 131072, dtype=np.int64)
    return DeviceWorkload(0, 0, lengths, cli=1, draw_latent=draw_latent)


def case_index_decode(reps):
    # as the decode step runs it: the scores and the top-k's first radix pass
    cfg = lsa.LsaConfig()
    wl = _decode_layer(False)
    scores = torch.empty((16, 131072), device="cuda")
    hist = lsa.topk_hist_buffer(16)
    for _ in range(reps):
        lsa.index_scores(cfg, wl.seq_of_row, wl.pos, wl.q_idx, wl.w, wl.k_idx, wl.k_off, 131072, scores,
                         topk_hist=hist)


def case_index_prefill(reps):
    cfg = lsa.LsaConfig()
    n = 16384
    wl = DeviceWorkload(0, 0, [n], n_rows=n, q_start=0, cli=1, draw_latent=False)
    scores = torch.empty((n, n), device="cuda")
    for _ in range(reps):
        lsa.index_scores(cfg, None, wl.pos, wl.q_idx, wl.w, wl.k_idx, None, n, scores)


def case_topk_decode(reps):
    cfg = lsa.LsaConfig()
    wl = _decode_layer(False)
    scores = torch.empty((16, 131072), device="cuda")
    hist = lsa.topk_hist_buffer(16)
    lsa.index_scores(cfg, wl.seq_of_row, wl.pos, wl.q_idx, wl.w, wl.k_idx, wl.k_off, 131072, scores,
                     topk_hist=hist)
    idx = torch.empty((16, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((16,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(cfg, lsa.OP_TOPK, 16, 16, 131072)
    for _ in range(reps):
        lsa.topk(cfg, wl.pos, 131072, scores, idx, cnt, ws, topk_hist=hist)


def case_topk_rows(reps):
    cfg = lsa.LsaConfig()
    n, L = 512, 500000
    scores = torch.empty((n, L), device="cuda")
    lsa.synth_normal_f32(scores, 0, 7)
    pos = torch.full((n,), L - 1, dtype=torch.int32, device="cuda")
    idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(cfg, lsa.OP_TOPK, n, n, L)
    for _ in range(reps):
        lsa.topk(cfg, pos, L, scores, idx, cnt, ws)


def case_mla_decode(reps):
    cfg = lsa.LsaConfig(cli_factor=1)
    wl = _decode_layer(True)
    rng = np.random.default_rng(0)
    idx = torch.from_numpy(np.stack([np.sort(rng.choice(131072, 2048, replace=False)) for _ in range(16)])
                           .astype(np.int32)).cuda()
    cnt = torch.full((16,), 2048, dtype=torch.int32, device="cuda")
    out = torch.empty((16, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((16, 32), device="cuda")
    ws = lsa.workspace(cfg, lsa.OP_MLA_DECODE, 16, 16, 131072)
    for _ in range(reps):
        lsa.sparse_mla_decode(cfg, wl.q_abs[0], wl.latent[0], wl.k_off, idx, cnt, 131072, out, lse, ws)


def case_mla_layer(reps):
    cfg = lsa.LsaConfig()
    lengths = np.full(16, 131072, dtype=np.int64)
    wl = DeviceWorkload(0, 0, lengths, cli=2)
    scores = torch.empty((16, 131072), device="cuda")
    hist = lsa.topk_hist_buffer(16)
    idx = torch.empty((16, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((16,), dtype=torch.int32, device="cuda")
    lsa.index_scores(cfg, wl.seq_of_row, wl.pos, wl.q_idx, wl.w, wl.k_idx, wl.k_off, 131072, scores, topk_hist=hist)
    lsa.topk(cfg, wl.pos, 131072, scores, idx, cnt, lsa.workspace(cfg, lsa.OP_TOPK, 16, 16, 131072), topk_hist=hist)
    outs = [torch.empty((16, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((16, 32), device="cuda") for _ in range(2)]
    ws = lsa.workspace(cfg, lsa.OP_MLA_DECODE_LAYER, 16, 16, 131072)
    for _ in range(reps):
        lsa.sparse_mla_decode_layer(cfg, wl.q_abs, wl.latent, wl.k_off, idx, cnt, 131072, outs, lses, ws)


def case_mla_prefill(reps):
    cfg = lsa.LsaConfig(cli_factor=1)
    n_keys, n_rows = 16384, 4096
    wl = DeviceWorkload(0, 0, [n_keys], n_rows=n_rows, q_start=n_keys - n_rows, cli=1)
    rng = np.random.default_rng(0)
    idx = torch.from_numpy(np.stack([np.sort(rng.choice(int(p) + 1, 2048, replace=False))
                                     for p in wl.pos.cpu().numpy()]).astype(np.int32)).cuda()
    cnt = torch.full((n_rows,), 2048, dtype=torch.int32, device="cuda")
    out = torch.empty((n_rows, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((n_rows, 32), device="cuda")
    ws = lsa.workspace(cfg, lsa.OP_MLA_PREFILL, n_rows, 1, n_keys)
    for _ in range(reps):
        lsa.sparse_mla_prefill(cfg, wl.pos, wl.q_abs[0], wl.latent[0], idx, cnt, out, lse, ws)


def case_decode_8k(reps):
    cfg = lsa.LsaConfig()
    wl = DeviceWorkload(0, 0, np.array([8192], dtype=np.int64))
    outs = [torch.empty((1, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((1, 32), device="cuda") for _ in range(2)]
    ws = lsa.workspace(cfg, lsa.OP_FORWARD_DECODE, 1, 1, 8192)
    for _ in range(reps):
        lsa.forward(cfg, 0, wl.seq_of_row, wl.pos, 8192, wl.q_idx, wl.w, wl.k_idx, wl.k_off, wl.q_abs, wl.latent,
                    outs, lses, ws)


def case_decode_1m(reps):
    cfg = lsa.LsaConfig()
    lengths = np.full(4, 983040, dtype=np.int64)
    wl = DeviceWorkload(0, 0, lengths)
    outs = [torch.empty((4, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((4, 32), device="cuda") for _ in range(2)]
    ws = lsa.workspace(cfg, lsa.OP_FORWARD_DECODE, 4, 4, 983040)
    for _ in range(reps):
        lsa.forward(cfg, 0, wl.seq_of_row, wl.pos, 983040, wl.q_idx, wl.w, wl.k_idx, wl.k_off, wl.q_abs, wl.latent,
                    outs, lses, ws)


def case_chunk_1m(reps):
    cfg = lsa.LsaConfig()
    n, q0 = 4096, 983040
    wl = DeviceWorkload(0, 0, [q0 + n], n_rows=n, q_start=q0)
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((n, 32), device="cuda") for _ in range(2)]
    ws = lsa.workspace(cfg, lsa.OP_FORWARD_PREFILL, n, 1, q0 + n)
    for _ in range(reps):
        lsa.forward(cfg, 1, None, wl.pos, q0 + n, wl.q_idx, wl.w, wl.k_idx, None, wl.q_abs, wl.latent, outs, lses,
                    ws)


def case_prefill_16k(reps):
    cfg = lsa.LsaConfig()
    n = 16384
    wl = DeviceWorkload(0, 0, [n], n_rows=n, q_start=0)
    scores = torch.empty((n, n), device="cuda")
    idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    tk_ws = lsa.workspace(cfg, lsa.OP_TOPK, n, 1, n)
    mla_ws = lsa.workspace(cfg, lsa.OP_MLA_PREFILL, n, 1, n)
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((n, 32), device="cuda") for _ in range(2)]
    for _ in range(reps):
        lsa.index_scores(cfg, None, wl.pos, wl.q_idx, wl.w, wl.k_idx, None, n, scores)
        lsa.topk(cfg, wl.pos, n, scores, idx, cnt, tk_ws)
        for z in range(2):
            lsa.sparse_mla_prefill(cfg, wl.pos, wl.q_abs[z], wl.latent[z], idx, cnt, outs[z], lses[z], mla_ws)


def case_hier_decode(reps):
    cfg = lsa.LsaConfig()
    wl = _decode_layer(False)
    block, n_blocks, B, ctx = 64, 128, 16, 131072
    blk_off = torch.tensor(lsa.block_offsets([ctx] * B, block), dtype=torch.int64, device="cuda")
    nb = ctx // block
    k_blk = torch.empty((B * nb, 128), dtype=torch.bfloat16, device="cuda")
    lsa.block_summaries(cfg, torch.arange(B, dtype=torch.int32, device="cuda").repeat_interleave(nb),
                        torch.arange(nb, dtype=torch.int32, device="cuda").repeat(B), wl.k_idx, wl.k_off, blk_off,
                        k_blk, block)
    new_seq = torch.arange(B, dtype=torch.int32, device="cuda")
    new_blk = torch.full((B,), nb - 1, dtype=torch.int32, device="cuda")
    idx = torch.empty((B, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B,), dtype=torch.int32, device="cuda")
    ws = lsa.hier_workspace(cfg, B, ctx, block, n_blocks)
    for _ in range(reps):
        lsa.block_summaries(cfg, new_seq, new_blk, wl.k_idx, wl.k_off, blk_off, k_blk, block)
        lsa.hier_select(cfg, wl.seq_of_row, wl.pos, wl.q_idx, wl.w, wl.k_idx, wl.k_off, k_blk, blk_off, ctx, idx,
                        cnt, ws, block, n_blocks)


CASES = {name[5:]: fn for name, fn in globals().items() if name.startswith("case_")}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=sorted(CASES))
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    lsa.load()
    CASES[args.case](args.reps)
    torch.cuda.synchronize()
    flags = lsa.device_error()
    if flags:
        print(f"device error flags 0x{flags:x}", file=sys.stderr)
        return 1
    print(f"{args.case}: ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
