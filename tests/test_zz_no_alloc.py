"""lsa_topk_static, the top-k entry point for callers that cannot allocate
device memory (graph capture, allocation-free serving loops, plugins given only
their buffers), must select exactly what lsa_topk selects with a caller
workspace, and exactly the oracle's set on the same fp32 scores, on consecutive
calls that share its built-in scratch.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import lsa_ref as R

pytestmark = pytest.mark.gpu

MAX_ROWS = 64


def _short_rows(seed):
    # 40 rows of mixed lengths (dense, just past topk, up to 150000 columns);
    # every fifth row rounded to integers (ties)
    rng = np.random.default_rng(seed)
    pos = np.concatenate([[0, 700, 2047, 2048, 2049, 5000], rng.integers(2100, 150000, 34)]).astype(np.int32)
    rows = []
    for r, p in enumerate(pos):
        v = rng.standard_normal(p + 1).astype(np.float32) * 8
        rows.append(np.round(v) if r % 5 == 0 else v)
    return pos, rows


def _full_rows(seed):
    # the row limit: 64 rows longer than 16384 columns, so the multi-CTA select
    # runs on the built-in scratch, which then holds exactly 4096 threshold-bin
    # candidates per row. Rows with heavy ties (integers in [-6, 6]) and rows
    # whose threshold bin holds 5000-9000 middle columns (some all equal)
    # overflow it and take the rescan branch.
    rng = np.random.default_rng(seed)
    pos = rng.integers(16500, 40000, MAX_ROWS).astype(np.int32)
    rows = []
    for r, p in enumerate(pos):
        v = rng.standard_normal(p + 1).astype(np.float32)
        if r % 3 == 0:
            v = np.round(v * 2).astype(np.float32)
        elif r % 3 == 1:
            cols = rng.choice(np.arange(16, p + 1 - 1024), int(rng.integers(5000, 9000)), replace=False)
            v[cols] = 100.0 if r % 2 else rng.uniform(96.0, 112.0, len(cols)).astype(np.float32)
        rows.append(v)
    return pos, rows


def _check_case(L, pos_h, rows, call):
    n, max_len = len(pos_h), int(pos_h.max()) + 1
    s_h = np.full((n, max_len), -np.inf, dtype=np.float32)
    for r, p in enumerate(pos_h):
        s_h[r, : p + 1] = rows[r]
    cfg = L.LsaConfig()
    ocfg = R.LsaConfig(index_topk=cfg.index_topk, index_init_tokens=cfg.index_init_tokens,
                       index_local_tokens=cfg.index_local_tokens, cli_factor=cfg.cli_factor)
    pos = torch.from_numpy(pos_h).cuda()
    scores = torch.from_numpy(s_h).cuda()
    ref_idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    ref_cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    ws = L.workspace(cfg, L.OP_TOPK, n, n, max_len)
    L.topk(cfg, pos, max_len, scores, ref_idx, ref_cnt, ws)
    idx = torch.full((n, 2048), -9, dtype=torch.int32, device="cuda")
    cnt = torch.full((n,), -9, dtype=torch.int32, device="cuda")
    st = L.topk_static(cfg, pos, max_len, scores, idx, cnt)
    assert st == (L.LSA_DENSE if max_len <= cfg.index_topk else L.LSA_OK)
    assert L.device_error() == 0
    a, b = ref_idx.cpu().numpy(), idx.cpu().numpy()
    np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt.cpu().numpy())
    for r, p in enumerate(pos_h):
        p = int(p)
        nsel = min(p + 1, cfg.index_topk)
        np.testing.assert_array_equal(np.sort(b[r]), np.sort(a[r]), err_msg=f"call {call} row {r} vs lsa_topk")
        # both sides decide on the same fp32 values (exact in fp64): the oracle's set, ties to the lower column
        exp, _ = R.select_topk(R.mask_and_force(rows[r].astype(np.float64), p, max_len, ocfg), p, ocfg)
        assert cnt[r] == nsel
        np.testing.assert_array_equal(np.sort(b[r, :nsel]), exp, err_msg=f"call {call} row {r} vs the oracle")


def test_topk_static_matches_topk_and_oracle_on_two_calls():
    from sparse_attention_03_b200 import lsa
    lsa.load()
    for call, seed in enumerate((1, 2)):
        _check_case(lsa, *_short_rows(seed), call)


def test_topk_static_at_the_row_limit_with_ties_and_overfull_bins():
    from sparse_attention_03_b200 import lsa
    lsa.load()
    for call, seed in enumerate((3, 4)):
        _check_case(lsa, *_full_rows(seed), call)


def test_topk_static_rejects_too_many_rows_and_bad_configs():
    from sparse_attention_03_b200 import lsa
    lib = lsa.load()
    cfg = lsa.LsaConfig().c()
    args = (ctypes.c_void_p(16), 5000, ctypes.c_void_p(16), 5000, ctypes.c_void_p(16), ctypes.c_void_p(16), None)
    assert lib.lsa_topk_static(ctypes.byref(cfg), MAX_ROWS + 1, *args) == lsa.LSA_ERR_INVALID
    assert b"exceed" in lib.lsa_last_error()
    bad = lsa.LsaConfig().c()
    bad.n_heads = 16          # a head shape the kernels do not implement: rejected as lsa_topk rejects it
    assert lib.lsa_topk_static(ctypes.byref(bad), 4, *args) == lsa.LSA_ERR_UNSUPPORTED
    bad = lsa.LsaConfig().c()
    bad.softmax_scale = 0.0
    assert lib.lsa_topk_static(ctypes.byref(bad), 4, *args) == lsa.LSA_ERR_INVALID
