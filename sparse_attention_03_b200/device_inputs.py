"""Synthetic LSA workloads drawn directly in device memory.

Shapes and tensor ids follow lsa_synth.Workload; the values come from the
library's own generator kernels (lsa_synth_* in include/lsa.h), which implement
the same counter-based definition, so any slice can be re-drawn on the host
bit for bit. Used for workloads too large to draw on the host (multi-GB caches).
"""
from __future__ import annotations

import numpy as np
import torch

import lsa_synth as S

from . import lsa


def _bf16(shape, device):
    return torch.empty(shape, dtype=torch.bfloat16, device=device)


class DeviceWorkload:
    """One layer's inputs on the device. Decode when n_rows is None, else prefill."""

    def __init__(self, seed: int, layer: int, lengths, n_rows=None, q_start=None, cli: int = 2,
                 device="cuda", draw_latent: bool = True):
        self.seed, self.layer, self.cli = seed, layer, cli
        self.lengths = np.asarray(lengths, dtype=np.int64)
        off = S.offsets(self.lengths)
        total = int(off[-1])
        self.total_keys = total
        if n_rows is None:
            self.mode = 0
            self.n_rows = len(self.lengths)
            self.pos = torch.from_numpy((self.lengths - 1).astype(np.int32)).to(device)
            self.seq_of_row = torch.arange(self.n_rows, dtype=torch.int32, device=device)
            self.k_off = torch.from_numpy(off).to(device)
        else:
            self.mode = 1
            self.n_rows = int(n_rows)
            self.pos = (int(q_start) + torch.arange(self.n_rows, dtype=torch.int32)).to(device)
            self.seq_of_row = None
            self.k_off = None
        self.max_len = int(self.lengths.max())
        R = self.n_rows
        self.q_idx = _bf16((R, S.HI, S.DI), device)
        lsa.synth_normal_bf16(self.q_idx, seed, S.tid(layer, S.Q_IDX))
        self.w = torch.empty((R, S.HI), dtype=torch.float32, device=device)
        lsa.synth_normal_f32(self.w, seed, S.tid(layer, S.W), sigma=float(S.W_SIGMA))
        self.k_idx = _bf16((total, S.DI), device)
        lsa.synth_rms_rows_bf16(self.k_idx, seed, S.tid(layer, S.K_IDX))
        self.q_abs = []
        self.latent = []
        for z in range(cli):
            q = _bf16((R, S.H, S.DLAT), device)
            lsa.synth_normal_bf16(q, seed, S.tid(layer, S.q_abs_kind(z)))
            self.q_abs.append(q)
            if draw_latent:
                c = _bf16((total, S.DLAT), device)
                lsa.synth_normal_bf16(c, seed, S.tid(layer, S.lat_kind(z)))
                self.latent.append(c)
