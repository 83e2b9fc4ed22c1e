"""GPU parity: every C-ABI entry point against the fp64 oracle on seeded inputs.

Inputs come from the host generator (lsa_synth) and are uploaded, or, for the
full-size workloads, are drawn on the device and the sampled rows re-drawn on
the host; no oracle input or expected value comes from the CUDA path.
"""
import numpy as np
import pytest
import torch

import lsa_synth as S
from lsa_testutil import (GAP_RTOL, assert_attention, assert_scores, bf16_dev, bf16_host_f64, check_selection,
                          f32_dev, host_rows, i32_dev, i64_dev, oracle_cfg)
from oracle import lsa_ref as R

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    from sparse_attention_03_b200 import lsa
    lsa.load()
    assert torch.cuda.is_available()
    return lsa


def _upload(wl: S.Workload):
    d = {}
    d["q_idx"] = bf16_dev(wl.q_idx)
    d["w"] = f32_dev(wl.w)
    d["k_idx"] = bf16_dev(wl.k_idx)
    d["q_abs"] = [bf16_dev(q) for q in wl.q_abs]
    d["latent"] = [bf16_dev(c) for c in wl.latent]
    d["pos"] = i32_dev(wl.pos)
    d["seq_of_row"] = i32_dev(wl.seq_of_row)
    d["k_off"] = i64_dev(wl.k_off)
    return d


# --------------------------------------------------------------------------
# Generator: the device kernels reproduce the host definition bit for bit.
# --------------------------------------------------------------------------
def test_device_generator_matches_host(L):
    x = torch.empty(100003, dtype=torch.bfloat16, device="cuda")
    L.synth_normal_bf16(x, 7, 21, first=12345)
    host = S.normal_bf16(7, 21, 12345, 100003)
    np.testing.assert_array_equal(x.view(torch.int16).cpu().numpy().view(np.uint16), host)
    y = torch.empty(5001, dtype=torch.float32, device="cuda")
    L.synth_normal_f32(y, 3, 4, first=99, sigma=float(S.W_SIGMA))
    np.testing.assert_array_equal(y.cpu().numpy(), S.normal_f32(3, 4, 99, 5001, S.W_SIGMA))
    k = torch.empty((777, 128), dtype=torch.bfloat16, device="cuda")
    L.synth_rms_rows_bf16(k, 0, 2, first_row=1000)
    np.testing.assert_array_equal(k.view(torch.int16).cpu().numpy().view(np.uint16),
                                  S.rms_rows_bf16(0, 2, 1000, 777, 128))


# --------------------------------------------------------------------------
# Indexer
# --------------------------------------------------------------------------
DECODE_LENGTHS = [1, 17, 1040, 1041, 2047, 2048, 2049, 3001, 5000, 8191, 12345]


def test_index_scores_decode_varlen(L):
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    wl = S.Workload(0, 0, DECODE_LENGTHS, cli=1)
    d = _upload(wl)
    max_len = int(max(DECODE_LENGTHS)) + 3
    ld = max_len + 5
    scores = torch.full((wl.n_rows, ld), float("nan"), device="cuda")
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], max_len, scores)
    assert L.device_error() == 0
    got = scores.cpu().numpy().astype(np.float64)
    for r in range(wl.n_rows):
        q, w, k, _, _ = host_rows(wl, r)
        assert_scores(got[r, :max_len], q, w, k, int(wl.pos[r]), ocfg, where=f"row {r}")
        assert np.isnan(got[r, int(wl.pos[r]) + 1:]).all(), "columns after pos must stay unwritten"


def test_index_scores_prefill_rows(L):
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    n = 3000
    wl = S.Workload(1, 0, [n], n_rows=n, q_start=0, cli=1)
    d = _upload(wl)
    scores = torch.empty((n, n), device="cuda")
    L.index_scores(cfg, None, d["pos"], d["q_idx"], d["w"], d["k_idx"], None, n, scores)
    assert L.device_error() == 0
    got = scores.cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(0)
    rows = sorted({0, 1, 15, 16, 1023, 1024, 2047, 2048, 2999} | set(rng.integers(0, n, 20).tolist()))
    for r in rows:
        q, w, k, _, _ = host_rows(wl, r)
        assert_scores(got[r], q, w, k, r, ocfg, where=f"row {r}")


def test_index_scores_prefill_streaming_path(L):
    # the same prefill rows through the streaming kernel (a sequence offset given)
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    n = 1500
    wl = S.Workload(1, 2, [n], n_rows=n, q_start=0, cli=1)
    d = _upload(wl)
    scores = torch.empty((n, n), device="cuda")
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], n, scores)
    got = scores.cpu().numpy().astype(np.float64)
    for r in (0, 17, 1039, 1040, 1499):
        q, w, k, _, _ = host_rows(wl, r)
        assert_scores(got[r], q, w, k, r, ocfg, where=f"row {r}")


@pytest.mark.parametrize("n_rows,n_keys,shuffle", [(1000, 1300, True), (16, 40000, False), (33, 777, True)])
def test_index_scores_tensor_core_shapes(L, n_rows, n_keys, shuffle):
    # ragged row blocks and key tiles, rows in any order, key-range splitting
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(n_rows)
    wl = S.Workload(3, 4, [n_keys], n_rows=n_rows, q_start=n_keys - n_rows, cli=1)
    pos = wl.pos.copy()
    if shuffle:
        pos = rng.permutation(np.arange(n_keys))[:n_rows].astype(np.int32)
    d = _upload(wl)
    ld = n_keys + 9
    scores = torch.full((n_rows, ld), float("nan"), device="cuda")
    L.device_error()
    L.index_scores(cfg, None, i32_dev(pos), d["q_idx"], d["w"], d["k_idx"], None, n_keys, scores)
    assert L.device_error() == 0
    got = scores.cpu().numpy().astype(np.float64)
    f = S.bf16_bits_to_f64
    k = f(wl.k_idx)
    rows = sorted(set(rng.integers(0, n_rows, 12).tolist()) | {0, n_rows - 1})
    for r in rows:
        assert_scores(got[r], f(wl.q_idx[r]), wl.w[r].astype(np.float64), k, int(pos[r]), ocfg, where=f"row {r}")
        assert np.isnan(got[r, pos[r] + 1:]).all(), "columns after pos must stay unwritten"


def test_index_scores_tiny_config_forcing(L):
    cfg = L.LsaConfig(index_topk=8, index_init_tokens=2, index_local_tokens=4)
    ocfg = oracle_cfg(cfg)
    wl = S.Workload(2, 0, [1, 3, 7, 8, 9, 20, 33], cli=1)
    d = _upload(wl)
    scores = torch.empty((wl.n_rows, 33), device="cuda")
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], 33, scores)
    got = scores.cpu().numpy().astype(np.float64)
    for r in range(wl.n_rows):
        q, w, k, _, _ = host_rows(wl, r)
        assert_scores(got[r], q, w, k, int(wl.pos[r]), ocfg, where=f"row {r}")


@pytest.mark.parametrize("streaming", [True, False])
def test_index_scores_many_rows_grid_chunks(L, streaming):
    # more than 65535 rows: the row-chunked streaming launch, and 4375 row blocks
    # of the tensor-core kernel
    cfg = L.LsaConfig()
    n_rows, n_keys = 70000, 40
    wl_q = S.normal_bf16(3, 0, 0, n_rows * 32 * 128).reshape(n_rows, 32, 128)
    w = S.normal_f32(3, 1, 0, n_rows * 32, S.W_SIGMA).reshape(n_rows, 32)
    k = S.rms_rows_bf16(3, 2, 0, n_keys, 128)
    pos = (np.arange(n_rows) % n_keys).astype(np.int32)
    scores = torch.empty((n_rows, n_keys), device="cuda")
    k_off = i64_dev(np.array([0, n_keys])) if streaming else None
    L.index_scores(cfg, None, i32_dev(pos), bf16_dev(wl_q), f32_dev(w), bf16_dev(k), k_off, n_keys, scores)
    got = scores.cpu().numpy().astype(np.float64)
    f = S.bf16_bits_to_f64
    for r in (0, 39, 65535, 65536, 69999):
        assert_scores(got[r], f(wl_q[r]), w[r].astype(np.float64), f(k), int(pos[r]), oracle_cfg(cfg))


# --------------------------------------------------------------------------
# Top-k on given fp32 scores: the decision is taken in fp32 on both sides, so
# the selection must match the oracle's exactly, ties included.
# --------------------------------------------------------------------------
def _topk_case(L, cfg, s_rows, pos, max_len, ld_pad=3):
    # ld_pad 3: rows not 16-byte aligned (4-byte loads); 0 with max_len % 4 == 0: 16-byte loads
    n_rows = len(pos)
    ld = max_len + ld_pad
    s = np.full((n_rows, ld), np.nan, dtype=np.float32)
    for r in range(n_rows):
        s[r, : pos[r] + 1] = s_rows[r][: pos[r] + 1]
        s[r, pos[r] + 1:max_len] = -np.inf
    ws = L.workspace(cfg, L.OP_TOPK, n_rows, 1, max_len)
    idx = torch.full((n_rows, cfg.index_topk), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((n_rows,), -7, dtype=torch.int32, device="cuda")
    st = L.topk(cfg, i32_dev(pos), max_len, f32_dev(s), idx, cnt, ws)
    return st, idx.cpu().numpy(), cnt.cpu().numpy()


def test_topk_exact_on_fp32_scores(L):
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(5)
    pos = np.array([0, 100, 2047, 2048, 2049, 3000, 20000, 70000, 250000, 9000], dtype=np.int64)
    max_len = int(pos.max()) + 1
    rows = []
    for i, p in enumerate(pos):
        if i == 7:
            v = rng.integers(-20, 20, p + 1).astype(np.float32)          # heavy ties
        elif i == 9:
            v = np.where(rng.random(p + 1) < 0.5, -0.0, 0.0).astype(np.float32)  # signed zeros
        else:
            v = rng.standard_normal(p + 1).astype(np.float32) * 8
        rows.append(v)
    st, idx, cnt = _topk_case(L, cfg, rows, pos, max_len)
    assert st == L.LSA_OK
    for r, p in enumerate(pos):
        s64 = R.mask_and_force(rows[r].astype(np.float64), int(p), max_len, ocfg)
        exp, dense = R.select_topk(s64, int(p), ocfg)
        n = int(p) + 1
        if dense:
            assert cnt[r] == n and np.array_equal(np.sort(idx[r, :n]), exp) and np.all(idx[r, n:] == -1)
        else:
            assert cnt[r] == cfg.index_topk
            np.testing.assert_array_equal(np.sort(idx[r]), exp, err_msg=f"row {r}")


@pytest.mark.parametrize("ld_pad", [0, 3])
def test_topk_many_long_rows_sampled_bound(L, ld_pad):
    # 256+ rows longer than 65536 middle columns take the one-CTA kernel's
    # sampled-bound path: a sample of the row sets a bound, one pass collects the
    # scores above it, the select finishes on them. Rows where the bound admits
    # too few (the best scores hidden between the sample runs) or too many (heavy
    # ties, all equal, an overfull bin) fall back to the exact two-pass path.
    # Exact sets against the oracle either way.
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(41 + ld_pad)
    n = 264
    pos = rng.integers(70000, 160000, n).astype(np.int64)
    if ld_pad == 0:
        pos -= (pos + 1) % 4          # 16-byte loads need max_len % 4 == 0 too
        pos = np.maximum(pos, 70000 - 1)
    rows = []
    for r, p in enumerate(pos):
        v = rng.standard_normal(p + 1).astype(np.float32)
        kind = r % 8
        if kind == 1:
            v = np.round(v * 2).astype(np.float32)                    # heavy ties: too many pass
        elif kind == 2:
            v[:] = 0.75                                               # all equal
        elif kind == 3:                                               # the best 1500 in one gap of the sample
            span = (p + 1 - 1024 - 16) - 256
            gap0 = 16 + span // 63 + 300
            v[gap0:gap0 + 1500] = 50.0 + rng.random(1500).astype(np.float32)
        elif kind == 4:                                               # an overfull bin
            cols = rng.choice(np.arange(16, p + 1 - 1024), 6000, replace=False)
            v[cols] = rng.uniform(96.0, 112.0, 6000).astype(np.float32)
        elif kind == 5:
            v *= 1e-3                                                 # tiny scores
        elif kind == 6:                                               # 600 large scores all inside the sample
            n_mid = (p + 1 - 1024) - 16                               # runs: the bound lands among them and
            for sg in range(60):                                      # admits fewer than the budget
                s0 = 16 + (n_mid - 256) * sg // 63
                v[s0 + 7:s0 + 247:24] = 50.0 + rng.random(10).astype(np.float32)
        rows.append(v)
    max_len = int(pos.max()) + 1 + (3 - int(pos.max()) % 4 if ld_pad == 0 else 0)
    st, idx, cnt = _topk_case(L, cfg, rows, pos, max_len, ld_pad)
    assert st == L.LSA_OK
    assert L.device_error() == 0
    for r, p in enumerate(pos):
        exp, dense = R.select_topk(R.mask_and_force(rows[r].astype(np.float64), int(p), max_len, ocfg), int(p), ocfg)
        assert cnt[r] == cfg.index_topk and not dense
        np.testing.assert_array_equal(np.sort(idx[r]), exp, err_msg=f"row {r} (kind {r % 8})")


def test_topk_all_equal_overflow_path(L):
    # all-equal scores overflow the candidate buffer and take the rescan path;
    # ties go to the lowest indices.
    cfg = L.LsaConfig()
    pos = np.array([150000, 4096], dtype=np.int64)
    rows = [np.full(p + 1, 1.5, dtype=np.float32) for p in pos]
    st, idx, cnt = _topk_case(L, cfg, rows, pos, int(pos.max()) + 1)
    for r, p in enumerate(pos):
        exp = np.sort(np.concatenate([np.arange(16), np.arange(16, 16 + 1008), np.arange(p + 1 - 1024, p + 1)]))
        np.testing.assert_array_equal(np.sort(idx[r]), exp)


def test_topk_multi_cta_long_rows(L):
    # few long rows take the multi-CTA kernels, including their rescan path when
    # the threshold bin overflows
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(21)
    pos = np.array([300000, 270001, 2048, 400000, 5000], dtype=np.int64)
    rows = [rng.standard_normal(pos[0] + 1).astype(np.float32) * 8,
            np.round(rng.standard_normal(pos[1] + 1) * 3).astype(np.float32),
            rng.standard_normal(pos[2] + 1).astype(np.float32),
            np.full(pos[3] + 1, 0.25, dtype=np.float32),
            rng.standard_normal(pos[4] + 1).astype(np.float32)]
    max_len = int(pos.max()) + 1
    st, idx, cnt = _topk_case(L, cfg, rows, pos, max_len)
    for r, p in enumerate(pos):
        exp, dense = R.select_topk(R.mask_and_force(rows[r].astype(np.float64), int(p), max_len, ocfg), int(p), ocfg)
        n = min(int(p) + 1, 2048)
        assert cnt[r] == n
        np.testing.assert_array_equal(np.sort(idx[r, :n]), exp, err_msg=f"row {r}")


def _dense_bin_rows(rng, pos, n_in_bin, exact=False):
    # N(0,1) scores with n_in_bin middle columns in [96, 112), one bin of the
    # first radix digit (sign, exponent and two mantissa bits), so the top of the
    # selection lands in an overfull threshold bin; exact=True puts them all at 100.
    rows = []
    for p, m in zip(pos, n_in_bin):
        v = rng.standard_normal(p + 1).astype(np.float32)
        cols = rng.choice(np.arange(16, p + 1 - 1024), m, replace=False)
        v[cols] = 100.0 if exact else rng.uniform(96.0, 112.0, m).astype(np.float32)
        rows.append(v)
    return rows


@pytest.mark.parametrize("kernel,ld_pad", [("per_row", 3), ("per_row", 0), ("multi_cta", 3)])
def test_topk_overfull_threshold_bin(L, kernel, ld_pad):
    # The threshold bin holds more candidates than shared memory: one more key
    # digit splits it (per-row kernel: over the row; multi-CTA kernel: over the
    # candidates held in the workspace), and when the split digit still
    # overflows (equal keys) the rescan path takes over. Exact sets.
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(31)
    if kernel == "per_row":   # rows of at most 16384 columns
        pos = np.array([15999, 12000, 16383, 9000], dtype=np.int64)
        rows = _dense_bin_rows(rng, pos[:2], [6000, 10900]) + \
            _dense_bin_rows(rng, pos[2:3], [7000], exact=True) + [np.full(pos[3] + 1, 1.5, dtype=np.float32)]
    else:                     # few long rows: candidate room of max_len / 16 per row
        pos = np.array([199999, 150000, 180000], dtype=np.int64)
        rows = _dense_bin_rows(rng, pos[:2], [7000, 12000]) + _dense_bin_rows(rng, pos[2:], [8000], exact=True)
    max_len = int(pos.max()) + 1
    st, idx, cnt = _topk_case(L, cfg, rows, pos, max_len, ld_pad)
    assert st == L.LSA_OK
    for r, p in enumerate(pos):
        exp, dense = R.select_topk(R.mask_and_force(rows[r].astype(np.float64), int(p), max_len, ocfg), int(p), ocfg)
        assert cnt[r] == cfg.index_topk and not dense
        np.testing.assert_array_equal(np.sort(idx[r]), exp, err_msg=f"{kernel} row {r}")
    assert L.device_error() == 0


def test_topk_overfull_bin_with_minimal_workspace(L):
    # a workspace of one base row block (4096 candidates per row) cannot hold the
    # overfull bin: the multi-CTA select falls back to rescanning the row, rows
    # one block at a time
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(37)
    pos = np.array([99999, 70000], dtype=np.int64)
    rows = _dense_bin_rows(rng, pos, [6000, 5000])
    max_len = int(pos.max()) + 1
    s = np.full((2, max_len), -np.inf, dtype=np.float32)
    for r, p in enumerate(pos):
        s[r, : p + 1] = rows[r]
    ws = torch.empty(40992 + 256, dtype=torch.uint8, device="cuda")
    idx = torch.empty((2, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((2,), dtype=torch.int32, device="cuda")
    assert L.topk(cfg, i32_dev(pos), max_len, f32_dev(s), idx, cnt, ws) == L.LSA_OK
    idx = idx.cpu().numpy()
    for r, p in enumerate(pos):
        exp, _ = R.select_topk(R.mask_and_force(s[r].astype(np.float64), int(p), max_len, ocfg), int(p), ocfg)
        np.testing.assert_array_equal(np.sort(idx[r]), exp, err_msg=f"row {r}")
    assert L.device_error() == 0


@pytest.mark.parametrize("streaming", [True, False])
def test_topk_with_indexer_histogram(L, streaming):
    # the histogram lsa_index_scores emits gives lsa_topk the same selection as
    # its own first pass (both indexer kernels: streaming, and tensor-core + one pass)
    cfg = L.LsaConfig()
    n = 6000
    wl = S.Workload(14, 0, [n], n_rows=300, q_start=n - 300, cli=1)
    d = _upload(wl)
    k_off = d["k_off"] if streaming else None
    seq = torch.zeros(300, dtype=torch.int32, device="cuda") if streaming else None
    scores = torch.empty((300, n), device="cuda")
    hist = L.topk_hist_buffer(300)
    L.index_scores(cfg, seq, d["pos"], d["q_idx"], d["w"], d["k_idx"], k_off, n, scores, topk_hist=hist)
    ws = L.workspace(cfg, L.OP_TOPK, 300, 1, n)
    outs = []
    for h in (hist, None):
        idx = torch.full((300, 2048), -3, dtype=torch.int32, device="cuda")
        cnt = torch.full((300,), -3, dtype=torch.int32, device="cuda")
        L.topk(cfg, d["pos"], n, scores, idx, cnt, ws, topk_hist=h)
        outs.append((np.sort(idx.cpu().numpy(), axis=1), cnt.cpu().numpy()))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    assert L.device_error() == 0


def test_topk_tiny_config_brute(L):
    cfg = L.LsaConfig(index_topk=8, index_init_tokens=2, index_local_tokens=4)
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(11)
    pos = np.array([0, 5, 7, 8, 9, 12, 30, 63], dtype=np.int64)
    rows = [rng.integers(-3, 4, p + 1).astype(np.float32) for p in pos]
    st, idx, cnt = _topk_case(L, cfg, rows, pos, 64)
    for r, p in enumerate(pos):
        s64 = R.mask_and_force(rows[r].astype(np.float64), int(p), 64, ocfg)
        exp, dense = R.select_topk(s64, int(p), ocfg)
        n = min(int(p) + 1, 8)
        assert cnt[r] == n
        np.testing.assert_array_equal(np.sort(idx[r, :n]), exp)


def test_topk_all_dense_status(L):
    cfg = L.LsaConfig()
    pos = np.array([0, 10, 2047], dtype=np.int64)
    rows = [np.zeros(p + 1, dtype=np.float32) for p in pos]
    st, idx, cnt = _topk_case(L, cfg, rows, pos, 2048)
    assert st == L.LSA_DENSE
    assert list(cnt) == [1, 11, 2048]


def test_topk_small_workspace_row_blocks(L):
    # a workspace for 3 rows forces several row blocks
    cfg = L.LsaConfig()
    rng = np.random.default_rng(2)
    pos = np.array([5000, 4000, 3000, 2500, 6000, 2049, 7000], dtype=np.int64)
    max_len = 7001
    s = np.full((len(pos), max_len), -np.inf, dtype=np.float32)
    for r, p in enumerate(pos):
        s[r, : p + 1] = rng.standard_normal(p + 1)
    from sparse_attention_03_b200.lsa import LsaError  # noqa: F401
    ws = torch.empty(3 * 40992 + 256, dtype=torch.uint8, device="cuda")
    idx = torch.empty((len(pos), 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((len(pos),), dtype=torch.int32, device="cuda")
    L.topk(cfg, i32_dev(pos), max_len, f32_dev(s), idx, cnt, ws)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    ocfg = oracle_cfg(cfg)
    for r, p in enumerate(pos):
        exp, _ = R.select_topk(R.mask_and_force(s[r].astype(np.float64), int(p), max_len, ocfg), int(p), ocfg)
        np.testing.assert_array_equal(np.sort(idx[r]), exp)


# --------------------------------------------------------------------------
# Sparse MLA on a given selection
# --------------------------------------------------------------------------
def _oracle_selection(wl, r, ocfg):
    q, w, k, qa, lat = host_rows(wl, r)
    p = int(wl.pos[r])
    s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
    sel, dense = R.select_topk(s, p, ocfg)
    return sel, dense, qa, lat


def test_mla_decode_on_selection(L):
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    lengths = [1, 64, 65, 2048, 2049, 5000, 9000, 4097]
    wl = S.Workload(4, 0, lengths, cli=1)
    d = _upload(wl)
    B = wl.n_rows
    idx = np.full((B, 2048), -1, dtype=np.int32)
    cnt = np.zeros(B, dtype=np.int32)
    exp = []
    for r in range(B):
        sel, dense, qa, lat = _oracle_selection(wl, r, ocfg)
        idx[r, : len(sel)] = np.random.default_rng(r).permutation(sel)  # order must not matter
        cnt[r] = len(sel)
        exp.append(R.mla(qa[0], lat[0][sel], ocfg))
    out = torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 32), device="cuda")
    for use_ws in (True, False):   # split-K + merge, and single pass
        ws = L.workspace(cfg, L.OP_MLA_DECODE, B, B, max(lengths)) if use_ws else None
        L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], i32_dev(idx), i32_dev(cnt),
                            max(lengths), out, lse, ws)
        assert L.device_error() == 0
        o, l = bf16_host_f64(out), lse.cpu().numpy()
        for r in range(B):
            assert_attention(o[r], l[r], exp[r][0], exp[r][1], where=f"row {r} ws={use_ws}")


def test_mla_rising_logits_rescale(L):
    # logits that keep rising from tile to tile by far more than 2^8 force the
    # attention kernel to rescale its running output; the oracle is exact fp64
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    rng = np.random.default_rng(17)
    n = 2048
    c = (rng.standard_normal((n, 576)) * 0.1).astype(np.float32)
    c[:, 0] = np.linspace(-40.0, 60.0, n)                      # logit driver along dim 0
    perm = rng.permutation(n)                                   # rising within the list order too
    q = (rng.standard_normal((32, 576)) * 0.05).astype(np.float32)
    q[:, 0] = 12.0
    c_bits, q_bits = S.f32_to_bf16_bits(c), S.f32_to_bf16_bits(q)
    idx = np.full((1, 2048), -1, dtype=np.int32)
    idx[0] = np.sort(perm)                                      # ascending = rising logits
    out = torch.empty((1, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 32), device="cuda")
    for ws in (None, L.workspace(cfg, L.OP_MLA_DECODE, 1, 1, n)):
        L.sparse_mla_decode(cfg, bf16_dev(q_bits[None]), bf16_dev(c_bits), i64_dev(np.array([0, n])),
                            i32_dev(idx), i32_dev(np.array([2048])), n, out, lse, ws)
        assert L.device_error() == 0
        eo, el = R.mla(S.bf16_bits_to_f64(q_bits), S.bf16_bits_to_f64(c_bits), ocfg)
        assert_attention(bf16_host_f64(out)[0], lse.cpu().numpy()[0], eo, el)


@pytest.mark.parametrize("pattern", [(16, 1024, 4096), (2, 3, 8), (0, 1, 1), (40, 100, 64), (5, 0, 300)])
def test_loza_decode_varlen(L, pattern):
    # LoZA rows of sequences whose lengths straddle the sink, the recent window and
    # chunk boundaries; split-K with a workspace and one pass without
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    pat = R.LozaPattern(*pattern)
    lengths = [1, 3, 16, 17, 300, 1024, 1025, 4095, 4096, 4097, 5121, 9000]
    wl = S.Workload(51, 0, lengths, cli=1)
    d = _upload(wl)
    B, max_len = len(lengths), max(lengths)
    f = S.bf16_bits_to_f64
    exp = []
    for b in range(B):
        a, e = int(wl.k_off[b]), int(wl.k_off[b + 1])
        exp.append(R.loza_row(f(wl.q_abs[0][b]), f(wl.latent[0][a:e]), int(wl.pos[b]), pat, ocfg))
    out = torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 32), device="cuda")
    for ws in (L.workspace(cfg, L.OP_MLA_DECODE, B, B, max_len), None):
        out.fill_(float("nan"))
        L.loza_mla(cfg, pattern, 0, d["seq_of_row"], d["pos"], d["k_off"], max_len, d["q_abs"][0], d["latent"][0],
                   out, lse, ws)
        assert L.device_error() == 0
        o, l = bf16_host_f64(out), lse.cpu().numpy()
        for b in range(B):
            assert_attention(o[b], l[b], exp[b][0], exp[b][1], where=f"{pattern} len {lengths[b]} ws={ws is not None}")


@pytest.mark.parametrize("pattern", [(16, 1024, 4096), (2, 3, 8), (16, 64, 256)])
def test_loza_prefill_rows(L, pattern):
    # a prefill chunk at an offset, rows crossing chunk boundaries
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    pat = R.LozaPattern(*pattern)
    n_keys, n_rows = 5200, 300
    wl = S.Workload(52, 0, [n_keys], n_rows=n_rows, q_start=n_keys - n_rows, cli=1)
    d = _upload(wl)
    out = torch.empty((n_rows, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((n_rows, 32), device="cuda")
    ws = L.workspace(cfg, L.OP_MLA_PREFILL, n_rows, 1, n_keys)
    L.loza_mla(cfg, pattern, 1, None, d["pos"], None, n_keys, d["q_abs"][0], d["latent"][0], out, lse, ws)
    assert L.device_error() == 0
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    f = S.bf16_bits_to_f64
    c = f(wl.latent[0])
    for r in (0, 1, 95, 96, 97, 150, 199, n_rows - 1):
        eo, el = R.loza_row(f(wl.q_abs[0][r]), c, int(wl.pos[r]), pat, ocfg)
        assert_attention(o[r], l[r], eo, el, where=f"{pattern} row {r}")


def test_loza_decode_explicit_positions(L):
    # rows that are not the last key of their sequence, in shuffled sequence order
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    pattern = (16, 256, 1024)
    lengths = [3000, 5000, 1500]
    wl = S.Workload(53, 0, lengths, cli=1)
    d = _upload(wl)
    seq = np.array([2, 0, 1, 1, 0], dtype=np.int32)
    pos = np.array([1499, 1023, 4095, 2000, 17], dtype=np.int32)
    q = S.normal_bf16(53, S.tid(9, S.Q_ABS0), 0, 5 * 32 * 576).reshape(5, 32, 576)
    out = torch.empty((5, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((5, 32), device="cuda")
    L.loza_mla(cfg, pattern, 0, i32_dev(seq), i32_dev(pos), d["k_off"], max(lengths), bf16_dev(q), d["latent"][0],
               out, lse, L.workspace(cfg, L.OP_MLA_DECODE, 5, 3, max(lengths)))
    assert L.device_error() == 0
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    f = S.bf16_bits_to_f64
    for r in range(5):
        a, e = int(wl.k_off[seq[r]]), int(wl.k_off[seq[r] + 1])
        eo, el = R.loza_row(f(q[r]), f(wl.latent[0][a:e]), int(pos[r]), R.LozaPattern(*pattern), ocfg)
        assert_attention(o[r], l[r], eo, el, where=f"row {r}")


def test_mla_decode_dense(L):
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    lengths = [1, 33, 700, 2048, 3000]
    wl = S.Workload(5, 0, lengths, cli=1)
    d = _upload(wl)
    out = torch.empty((len(lengths), 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((len(lengths), 32), device="cuda")
    ws = L.workspace(cfg, L.OP_MLA_DECODE, len(lengths), len(lengths), max(lengths))
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], None, None, max(lengths), out, lse, ws)
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    for r in range(len(lengths)):
        _, _, _, qa, lat = host_rows(wl, r)
        eo, el = R.dense_mla_row(qa[0], lat[0], lengths[r] - 1, ocfg)
        assert_attention(o[r], l[r], eo, el, where=f"row {r}")


def test_mla_decode_dense_many_splits(L):
    # a long dense list splits beyond one cluster (more than 8 CTAs per row), so
    # the partials go through the workspace and the merge kernel
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    lengths = [20000, 9000]
    wl = S.Workload(18, 0, lengths, cli=1)
    d = _upload(wl)
    out = torch.empty((2, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 32), device="cuda")
    ws = L.workspace(cfg, L.OP_MLA_DECODE, 2, 2, max(lengths))
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], None, None, max(lengths), out, lse, ws)
    assert L.device_error() == 0
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    for r in range(2):
        _, _, _, qa, lat = host_rows(wl, r)
        eo, el = R.dense_mla_row(qa[0], lat[0], lengths[r] - 1, ocfg)
        assert_attention(o[r], l[r], eo, el, where=f"row {r}")


def test_mla_prefill_on_selection(L):
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    n = 2600
    wl = S.Workload(6, 0, [n], n_rows=n, q_start=0, cli=1)
    d = _upload(wl)
    rows = [0, 1, 100, 2046, 2047, 2048, 2049, 2599]
    sub = np.array(rows)
    idx = np.full((len(rows), 2048), -1, dtype=np.int32)
    cnt = np.zeros(len(rows), dtype=np.int32)
    exp = []
    for i, r in enumerate(rows):
        sel, dense, qa, lat = _oracle_selection(wl, r, ocfg)
        idx[i, : len(sel)] = sel
        cnt[i] = len(sel)
        exp.append(R.mla(qa[0], lat[0][sel], ocfg))
    out = torch.empty((len(rows), 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((len(rows), 32), device="cuda")
    q_sub = d["q_abs"][0][torch.from_numpy(sub).cuda()].contiguous()
    L.sparse_mla_prefill(cfg, i32_dev(sub), q_sub, d["latent"][0], i32_dev(idx), i32_dev(cnt), out, lse, None)
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    for i in range(len(rows)):
        assert_attention(o[i], l[i], exp[i][0], exp[i][1], where=f"row {rows[i]}")


def test_mla_bad_index_is_flagged_not_faulting(L):
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    wl = S.Workload(7, 0, [3000], cli=1)
    d = _upload(wl)
    sel = np.arange(0, 3000, 2)[:1000].astype(np.int32)
    bad = sel.copy()
    bad[5] = 10 ** 9          # far outside the sequence
    bad[6] = -3
    idx = np.full((1, 2048), -1, dtype=np.int32)
    idx[0, :1000] = bad
    out = torch.empty((1, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 32), device="cuda")
    L.device_error()
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], i32_dev(idx), i32_dev(np.array([1000])),
                        3000, out, lse, None)
    assert L.device_error() & L.DEVERR_INDEX
    _, _, _, qa, lat = host_rows(wl, 0)
    keep = np.delete(sel, [5, 6])
    eo, el = R.mla(qa[0], lat[0][keep], ocfg)
    assert_attention(bf16_host_f64(out)[0], lse.cpu().numpy()[0], eo, el)


# --------------------------------------------------------------------------
# Whole layer through lsa_forward
# --------------------------------------------------------------------------
def _forward_check(L, wl, d, cfg, mode, rows_to_check, max_len):
    ocfg = oracle_cfg(cfg)
    n = wl.n_rows
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(cfg.cli_factor)]
    lses = [torch.empty((n, 32), device="cuda") for _ in range(cfg.cli_factor)]
    idx = torch.full((n, cfg.index_topk), -5, dtype=torch.int32, device="cuda")
    cnt = torch.full((n,), -5, dtype=torch.int32, device="cuda")
    op = L.OP_FORWARD_DECODE if mode == 0 else L.OP_FORWARD_PREFILL
    ws = L.workspace(cfg, op, n, len(wl.lengths), max_len)
    L.forward(cfg, mode, d["seq_of_row"] if mode == 0 else None, d["pos"], max_len, d["q_idx"], d["w"],
              d["k_idx"], d["k_off"] if mode == 0 else None, d["q_abs"], d["latent"], outs, lses, ws,
              idx_out=idx, count_out=cnt)
    assert L.device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    o = [bf16_host_f64(t) for t in outs]
    l = [t.cpu().numpy() for t in lses]
    dense_all = max_len <= cfg.index_topk
    for r in rows_to_check:
        q, w, k, qa, lat = host_rows(wl, r)
        p = int(wl.pos[r])
        sel, dense, res = R.lsa_row(q, w, k, p, qa, lat, ocfg)
        exact = True
        if not dense_all:
            s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
            exact = check_selection(idx[r], int(cnt[r]), s, p, ocfg, where=f"row {r}")
        for z in range(cfg.cli_factor):
            assert_attention(o[z][r], l[z][r], res[z][0], res[z][1], check_lse=exact, where=f"row {r} sub {z}")


def test_forward_decode_varlen(L):
    cfg = L.LsaConfig()
    lengths = [2049, 3000, 4100, 5555, 7000, 8192, 2100, 6100]
    wl = S.Workload(8, 3, lengths)
    _forward_check(L, wl, _upload(wl), cfg, 0, range(len(lengths)), max(lengths))


def test_forward_decode_dense_fallback(L):
    cfg = L.LsaConfig()
    lengths = [1, 100, 2048, 1500]
    wl = S.Workload(9, 0, lengths)
    _forward_check(L, wl, _upload(wl), cfg, 0, range(len(lengths)), max(lengths))


def test_forward_prefill(L):
    cfg = L.LsaConfig()
    n = 2700
    wl = S.Workload(10, 1, [n], n_rows=n, q_start=0)
    rng = np.random.default_rng(1)
    rows = sorted({0, 2047, 2048, 2049, n - 1} | set(rng.integers(2048, n, 6).tolist()) | {5, 700})
    _forward_check(L, wl, _upload(wl), cfg, 1, rows, n)


def test_forward_prefill_chunk_at_offset(L):
    # a chunk of new rows appended to a longer cache (rows see q_start + t)
    cfg = L.LsaConfig()
    n_keys, n_rows = 4000, 300
    wl = S.Workload(11, 0, [n_keys], n_rows=n_rows, q_start=n_keys - n_rows)
    _forward_check(L, wl, _upload(wl), cfg, 1, [0, 1, 150, 299], n_keys)


def test_forward_tiny_config(L):
    cfg = L.LsaConfig(index_topk=8, index_init_tokens=2, index_local_tokens=4)
    lengths = [1, 5, 8, 9, 10, 31, 64, 100]
    wl = S.Workload(12, 0, lengths)
    _forward_check(L, wl, _upload(wl), cfg, 0, range(len(lengths)), max(lengths))


def _mtp_case(L, seed, lengths, short=(), n_draft=3):
    # sequence b's index owner (the first draft step) sits at lengths[b] - n_draft,
    # so the cache holds the later drafts' keys; rows in `short` sit one position
    # later (the last draft's key is missing: flagged, not attended)
    cfg = L.LsaConfig(cli_factor=1)
    wl = S.Workload(seed, 0, lengths, cli=1)
    wl.pos = np.array([n - n_draft + (1 if b in short else 0) for b, n in enumerate(wl.lengths)], dtype=np.int32)
    d = _upload(wl)
    B, max_len = wl.n_rows, max(lengths)
    q_steps = [S.normal_bf16(seed, S.tid(50 + st, S.Q_ABS0), 0, B * 32 * 576).reshape(B, 32, 576)
               for st in range(n_draft)]
    scores = torch.empty((B, max_len), device="cuda")
    idx = torch.empty((B, cfg.index_topk), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B,), dtype=torch.int32, device="cuda")
    hist = L.topk_hist_buffer(B)
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], max_len, scores,
                   topk_hist=hist)
    L.topk(cfg, d["pos"], max_len, scores, idx, cnt, L.workspace(cfg, L.OP_TOPK, B, B, max_len), topk_hist=hist)
    outs = [torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(n_draft)]
    lses = [torch.empty((B, 32), device="cuda") for _ in range(n_draft)]
    L.mtp_mla_decode(cfg, d["pos"], [bf16_dev(q) for q in q_steps], d["latent"][0], d["k_off"], idx, cnt, max_len,
                     outs, lses, L.workspace(cfg, L.OP_MTP_DECODE, B, B, max_len))
    return cfg, wl, q_steps, idx.cpu().numpy(), cnt.cpu().numpy(), [(bf16_host_f64(o), l.cpu().numpy())
                                                                      for o, l in zip(outs, lses)]


def test_mtp_draft_steps_share_one_index_pass(L):
    # [LSA-2.0] "多token预测模块集成": the three MTP draft steps share one index
    # pass; one launch attends all three (oracle.mtp_round: step i sees the shared
    # selection plus keys p+1 .. p+i). Rows: sparse, the dense boundary (p + 1 =
    # 2048 and 2049), dense, long.
    lengths = [2052, 3000, 5002, 9001, 2050, 2051, 700, 12000]
    cfg, wl, q_steps, gi, gc, got = _mtp_case(L, 21, lengths)
    assert L.device_error() == 0
    ocfg = oracle_cfg(cfg)
    for r in range(wl.n_rows):
        q, w, k, _, lat = host_rows(wl, r)
        p = int(wl.pos[r])
        s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
        exact = check_selection(gi[r], int(gc[r]), s, p, ocfg, where=f"row {r}")
        qs = [S.bf16_bits_to_f64(q_steps[st][r]) for st in range(3)]
        sel, dense, res = R.mtp_round(q, w, k, p, qs, lat[0], ocfg)
        if not exact:   # a near-tie: the GPU's own (valid) set, through the same round
            sel = np.sort(gi[r, : gc[r]]).astype(np.int64)
            res = [R.mla(qs[st], lat[0][np.concatenate([sel, np.arange(p + 1, p + 1 + st)])], ocfg)
                   for st in range(3)]
        for st in range(3):
            assert_attention(got[st][0][r], got[st][1][r], res[st][0], res[st][1], where=f"row {r} step {st}")


@pytest.mark.parametrize("n_draft", [1, 2, 4])
def test_mtp_other_draft_counts(L, n_draft):
    # one draft step is the plain layer path over the selection; four is the
    # entry point's limit (three newer keys for the last step)
    lengths = [2600, 2049 + n_draft - 1, 5000, 1500]
    cfg, wl, q_steps, gi, gc, got = _mtp_case(L, 30 + n_draft, lengths, n_draft=n_draft)
    assert L.device_error() == 0
    ocfg = oracle_cfg(cfg)
    for r in range(wl.n_rows):
        q, w, k, _, lat = host_rows(wl, r)
        p = int(wl.pos[r])
        s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
        exact = check_selection(gi[r], int(gc[r]), s, p, ocfg, where=f"row {r}")
        qs = [S.bf16_bits_to_f64(q_steps[st][r]) for st in range(n_draft)]
        sel, _, res = R.mtp_round(q, w, k, p, qs, lat[0], ocfg)
        if not exact:
            sel = np.sort(gi[r, : gc[r]]).astype(np.int64)
            res = [R.mla(qs[st], lat[0][np.concatenate([sel, np.arange(p + 1, p + 1 + st)])], ocfg)
                   for st in range(n_draft)]
        for st in range(n_draft):
            assert_attention(got[st][0][r], got[st][1][r], res[st][0], res[st][1], where=f"row {r} step {st}")


def test_mla_decode_layer_single_sub_block_equals_topk_call(L):
    # with cli_factor 1 the layer call is lsa_sparse_mla_decode_topk: the same kernel
    # and split, so the same bits
    cfg = L.LsaConfig(cli_factor=1)
    lengths = [3000, 2048, 7000, 12]
    wl = S.Workload(26, 0, lengths, cli=1)
    d = _upload(wl)
    B, max_len = wl.n_rows, max(lengths)
    idx, cnt = _topk_lists(L, cfg, wl, d, max_len)
    ws = L.workspace(cfg, L.OP_MLA_DECODE_LAYER, B, B, max_len)
    o1, l1 = torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda"), torch.empty((B, 32), device="cuda")
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    L.sparse_mla_decode_layer(cfg, d["q_abs"], d["latent"], d["k_off"], idx, cnt, max_len, [o1], [l1], ws)
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], idx, cnt, max_len, o2, l2, ws,
                        lists_from_topk=True)
    assert L.device_error() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_mtp_draft_key_past_the_sequence_is_flagged(L):
    # the last draft's key is not in the cache: LSA_DEVERR_POS, and that step
    # attends to the keys that are there
    lengths = [3000, 2600]
    cfg, wl, q_steps, gi, gc, got = _mtp_case(L, 22, lengths, short=(1,))
    assert L.device_error() & L.DEVERR_POS
    ocfg = oracle_cfg(cfg)
    q, w, k, _, lat = host_rows(wl, 1)
    p = int(wl.pos[1])
    sel = np.sort(gi[1, : gc[1]]).astype(np.int64)
    eo, el = R.mla(S.bf16_bits_to_f64(q_steps[2][1]), lat[0][np.concatenate([sel, [p + 1]])], ocfg)
    assert_attention(got[2][0][1], got[2][1][1], eo, el, where="short row, step 2")


def test_mla_decode_layer_one_launch_matches_oracle(L):
    # both sub-blocks of a layer over one top-k selection in one launch (with
    # the in-kernel split-K merge), against the oracle's layer path
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    lengths = [2049, 3000, 4100, 5555, 7000, 8192, 2100, 6100, 1500, 16]
    wl = S.Workload(23, 0, lengths)
    d = _upload(wl)
    B, max_len = wl.n_rows, max(lengths)
    scores = torch.empty((B, max_len), device="cuda")
    idx = torch.empty((B, cfg.index_topk), dtype=torch.int32, device="cuda")
    cnt = torch.empty((B,), dtype=torch.int32, device="cuda")
    hist = L.topk_hist_buffer(B)
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], max_len, scores,
                   topk_hist=hist)
    L.topk(cfg, d["pos"], max_len, scores, idx, cnt, L.workspace(cfg, L.OP_TOPK, B, B, max_len), topk_hist=hist)
    outs = [torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((B, 32), device="cuda") for _ in range(2)]
    ws = L.workspace(cfg, L.OP_MLA_DECODE_LAYER, B, B, max_len)
    ws.random_(0, 256)   # the workspace needs no clearing
    for _ in range(2):   # and a second launch reuses it
        L.sparse_mla_decode_layer(cfg, d["q_abs"], d["latent"], d["k_off"], idx, cnt, max_len, outs, lses, ws)
        assert L.device_error() == 0
        gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
        o = [bf16_host_f64(t) for t in outs]
        l = [t.cpu().numpy() for t in lses]
        for r in range(B):
            q, w, k, qa, lat = host_rows(wl, r)
            p = int(wl.pos[r])
            s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
            exact = check_selection(gi[r], int(gc[r]), s, p, ocfg, where=f"row {r}")
            sel = R.select_topk(s, p, ocfg)[0] if exact else np.sort(gi[r, : gc[r]]).astype(np.int64)
            for z in range(2):
                eo, el = R.mla(qa[z], lat[z][sel], ocfg)
                assert_attention(o[z][r], l[z][r], eo, el, where=f"row {r} sub {z}")


def test_mla_topk_lists_wait_timeout_is_reported_and_the_next_call_is_clean(L):
    # the same for the attention over the top-k's lists (the tensor-core kernel):
    # every CTA's gather stops before its second tile, the waits give up after
    # 2 ms, the kernel still frees its tensor memory and returns
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    lengths = [3000, 5000, 2500, 7000, 1500]
    wl = S.Workload(25, 0, lengths, cli=1)
    d = _upload(wl)
    B, max_len = wl.n_rows, max(lengths)
    idx, cnt = _topk_lists(L, cfg, wl, d, max_len)
    out = torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 32), device="cuda")
    ws = L.workspace(cfg, L.OP_MLA_DECODE, B, B, max_len)
    L.debug_arm_mla_wait_test(2_000_000, 1)
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], idx, cnt, max_len, out, lse, ws,
                        lists_from_topk=True)
    assert L.device_error() & L.DEVERR_TIMEOUT
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], idx, cnt, max_len, out, lse, ws,
                        lists_from_topk=True)
    assert L.device_error() == 0
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    for r in range(B):
        q, w, k, qa, lat = host_rows(wl, r)
        p = int(wl.pos[r])
        s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
        exact = check_selection(gi[r], int(gc[r]), s, p, ocfg, where=f"row {r}")
        sel = R.select_topk(s, p, ocfg)[0] if exact else np.sort(gi[r, : gc[r]]).astype(np.int64)
        eo, el = R.mla(qa[0], lat[0][sel], ocfg)
        assert_attention(o[r], l[r], eo, el, where=f"row {r} after the timeout")


def test_mla_wait_timeout_is_reported_and_the_next_call_is_clean(L):
    # A bounded wait that runs out: the test hook makes every CTA's producer stop
    # before its second tile and the attention warps give up after 2 ms. The
    # kernel must return, report LSA_DEVERR_TIMEOUT, and leave the device fit for
    # the next call, which must match the oracle again.
    cfg = L.LsaConfig(cli_factor=1)
    ocfg = oracle_cfg(cfg)
    lengths = [3000, 5000, 2500, 7000]
    wl = S.Workload(24, 0, lengths, cli=1)
    d = _upload(wl)
    B, max_len = wl.n_rows, max(lengths)
    out = torch.empty((B, 32, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 32), device="cuda")
    ws = L.workspace(cfg, L.OP_MLA_DECODE, B, B, max_len)
    L.debug_arm_mla_wait_test(2_000_000, 1)
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], None, None, max_len, out, lse, ws)
    assert L.device_error() & L.DEVERR_TIMEOUT
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], None, None, max_len, out, lse, ws)
    assert L.device_error() == 0
    o, l = bf16_host_f64(out), lse.cpu().numpy()
    for r in range(B):
        _, _, _, qa, lat = host_rows(wl, r)
        eo, el = R.mla(qa[0], lat[0], ocfg)
        assert_attention(o[r], l[r], eo, el, where=f"row {r} after the timeout")


def test_empty_batch_is_noop(L):
    cfg = L.LsaConfig()
    e = torch.empty((0,), dtype=torch.int32, device="cuda")
    assert L.index_scores(cfg, None, e, torch.empty((0, 32, 128), dtype=torch.bfloat16, device="cuda"),
                          torch.empty((0, 32), device="cuda"),
                          torch.empty((8, 128), dtype=torch.bfloat16, device="cuda"), None, 8,
                          torch.empty((0, 8), device="cuda")) == 0


def test_position_past_sequence_is_flagged(L):
    cfg = L.LsaConfig()
    wl = S.Workload(13, 0, [100, 200], cli=1)
    d = _upload(wl)
    pos = i32_dev(np.array([99, 250]))    # row 1 claims position 250 in a 200-key sequence
    scores = torch.empty((2, 300), device="cuda")
    L.device_error()
    L.index_scores(cfg, d["seq_of_row"], pos, d["q_idx"], d["w"], d["k_idx"], d["k_off"], 300, scores)
    assert L.device_error() & L.DEVERR_POS


# --------------------------------------------------------------------------
# Full-size workloads (device-drawn), sampled rows against the oracle
# --------------------------------------------------------------------------
def _oracle_row_from_stream(seed, layer, k_off, b, p, cfg, cli=2):
    """The oracle on row b of a device-drawn decode workload, re-drawing inputs on the host."""
    ocfg = oracle_cfg(cfg)
    f = S.bf16_bits_to_f64
    a, e = int(k_off[b]), int(k_off[b + 1])
    q = f(S.normal_bf16(seed, S.tid(layer, S.Q_IDX), b * 4096, 4096)).reshape(32, 128)
    w = S.normal_f32(seed, S.tid(layer, S.W), b * 32, 32, S.W_SIGMA).astype(np.float64)
    k = f(S.rms_rows_bf16(seed, S.tid(layer, S.K_IDX), a, e - a, 128))
    s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, e - a, ocfg)
    sel, dense = R.select_topk(s, p, ocfg)
    res = []
    for z in range(cli):
        qa = f(S.normal_bf16(seed, S.tid(layer, S.q_abs_kind(z)), b * 32 * 576, 32 * 576)).reshape(32, 576)
        c = f(S.normal_bf16_rows(seed, S.tid(layer, S.lat_kind(z)), a + sel, 576))
        res.append(R.mla(qa, c, ocfg))
    return s, sel, res


@pytest.mark.parametrize("name,batch,lo,hi,sample", [
    ("decode_b64_16k_32k", 64, 16384, 32768, (0, 17, 63)),
    ("decode_b16_128k", 16, 131072, 131072, (3, 15)),
    ("decode_b4_983040", 4, 983040, 983040, (2,)),
])
def test_full_size_decode_sampled(L, name, batch, lo, hi, sample):
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    lengths = S.decode_lengths(0, batch, lo, hi)
    wl = DeviceWorkload(0, 0, lengths)
    n = wl.n_rows
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((n, 32), device="cuda") for _ in range(2)]
    idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    ws = L.workspace(cfg, L.OP_FORWARD_DECODE, n, n, wl.max_len)
    L.forward(cfg, 0, wl.seq_of_row, wl.pos, wl.max_len, wl.q_idx, wl.w, wl.k_idx, wl.k_off, wl.q_abs,
              wl.latent, outs, lses, ws, idx_out=idx, count_out=cnt)
    assert L.device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    k_off = S.offsets(lengths)
    for b in sample:
        p = int(lengths[b]) - 1
        s, sel, res = _oracle_row_from_stream(0, 0, k_off, b, p, cfg)
        exact = check_selection(idx[b], int(cnt[b]), s, p, ocfg, where=f"{name} row {b}")
        for z in range(2):
            assert_attention(bf16_host_f64(outs[z][b]), lses[z][b].cpu().numpy(), res[z][0], res[z][1],
                             check_lse=exact, where=f"{name} row {b} sub {z}")
    del wl
    torch.cuda.empty_cache()


def test_full_size_prefill_16k_sampled(L):
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    n = 16384
    wl = DeviceWorkload(0, 0, [n], n_rows=n, q_start=0)
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((n, 32), device="cuda") for _ in range(2)]
    idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    ws = L.workspace(cfg, L.OP_FORWARD_PREFILL, n, 1, n)
    L.forward(cfg, 1, None, wl.pos, n, wl.q_idx, wl.w, wl.k_idx, None, wl.q_abs, wl.latent, outs, lses, ws,
              idx_out=idx, count_out=cnt)
    assert L.device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    f = S.bf16_bits_to_f64
    k = f(S.rms_rows_bf16(0, S.tid(0, S.K_IDX), 0, n, 128))
    for r in (0, 2047, 2048, 9000, n - 1):
        q = f(S.normal_bf16(0, S.tid(0, S.Q_IDX), r * 4096, 4096)).reshape(32, 128)
        w = S.normal_f32(0, S.tid(0, S.W), r * 32, 32, S.W_SIGMA).astype(np.float64)
        s = R.mask_and_force(R.score_row(q, w, k[: r + 1]), r, n, ocfg)
        exact = check_selection(idx[r], int(cnt[r]), s, r, ocfg, where=f"prefill row {r}")
        sel, _ = R.select_topk(s, r, ocfg)
        for z in range(2):
            qa = f(S.normal_bf16(0, S.tid(0, S.q_abs_kind(z)), r * 32 * 576, 32 * 576)).reshape(32, 576)
            c = f(S.normal_bf16_rows(0, S.tid(0, S.lat_kind(z)), sel, 576))
            eo, el = R.mla(qa, c, ocfg)
            assert_attention(bf16_host_f64(outs[z][r]), lses[z][r].cpu().numpy(), eo, el, check_lse=exact,
                             where=f"prefill row {r} sub {z}")


def test_full_size_prefill_chunk_1m_sampled(L):
    # The long-context workload's prefill chunk: 4096 new rows at positions
    # 983040 .. 987135 against the whole 987136-key cache (every row sparse).
    # The 16 GB score matrix, the tensor-core indexer over 33 TFLOP of causal
    # pairs, the one-CTA-per-row top-k over 987136 columns and the prefill MLA
    # gathering from a 1.1 GB latent cache, sampled rows against the oracle.
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    n, q0 = 4096, 983040
    n_keys = q0 + n
    wl = DeviceWorkload(0, 0, [n_keys], n_rows=n, q_start=q0)
    outs = [torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    lses = [torch.empty((n, 32), device="cuda") for _ in range(2)]
    idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    ws = L.workspace(cfg, L.OP_FORWARD_PREFILL, n, 1, n_keys)
    L.forward(cfg, 1, None, wl.pos, n_keys, wl.q_idx, wl.w, wl.k_idx, None, wl.q_abs, wl.latent, outs, lses, ws,
              idx_out=idx, count_out=cnt)
    assert L.device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    del ws, wl
    torch.cuda.empty_cache()
    f = S.bf16_bits_to_f64
    k = f(S.rms_rows_bf16(0, S.tid(0, S.K_IDX), 0, n_keys, 128))
    for t in (0, 2049, n - 1):
        p = q0 + t
        q = f(S.normal_bf16(0, S.tid(0, S.Q_IDX), t * 4096, 4096)).reshape(32, 128)
        w = S.normal_f32(0, S.tid(0, S.W), t * 32, 32, S.W_SIGMA).astype(np.float64)
        s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, n_keys, ocfg)
        exact = check_selection(idx[t], int(cnt[t]), s, p, ocfg, where=f"chunk row {t}")
        sel, _ = R.select_topk(s, p, ocfg)
        for z in range(2):
            qa = f(S.normal_bf16(0, S.tid(0, S.q_abs_kind(z)), t * 32 * 576, 32 * 576)).reshape(32, 576)
            c = f(S.normal_bf16_rows(0, S.tid(0, S.lat_kind(z)), sel, 576))
            eo, el = R.mla(qa, c, ocfg)
            assert_attention(bf16_host_f64(outs[z][t]), lses[z][t].cpu().numpy(), eo, el, check_lse=exact,
                             where=f"chunk row {t} sub {z}")


# --------------------------------------------------------------------------
# The indexer's own projections and the key-cache append (upstream of the path)
# --------------------------------------------------------------------------
def _project_inputs(seed, n_rows, q_lora=1536, hidden=3072):
    f = S.bf16_bits_to_f64
    c_q = S.normal_bf16(seed, S.tid(0, S.C_Q), 0, n_rows * q_lora).reshape(n_rows, q_lora)
    h = S.normal_bf16(seed, S.tid(0, S.HIDDEN), 0, n_rows * hidden).reshape(n_rows, hidden)
    wq_b = S.normal_bf16(seed, S.tid(0, S.WQ_B), 0, 4096 * q_lora, 1 / np.sqrt(q_lora)).reshape(4096, q_lora)
    wk = S.normal_bf16(seed, S.tid(0, S.WK), 0, 128 * hidden, 1 / np.sqrt(hidden)).reshape(128, hidden)
    wp = S.normal_bf16(seed, S.tid(0, S.WPROJ), 0, 32 * hidden, 1 / np.sqrt(hidden)).reshape(32, hidden)
    g = S.f32_to_bf16_bits((1.0 + 0.1 * f(S.normal_bf16(seed, S.tid(0, S.KNORM), 0, 128))).astype(np.float32))
    return c_q, h, wq_b, wk, wp, g


def _pair_bound(m):
    # |error| after RoPE of a pair (a, b) is at most the sum of both inputs' errors
    m = m.copy()
    a, b = m[..., 64:96].copy(), m[..., 96:].copy()
    m[..., 64:96] = a + b
    m[..., 96:] = a + b
    return m


def _check_bf16(got, exp, mag, where):
    # bf16 output: one bf16 ulp (2^-8 relative) of rounding plus the fp32
    # accumulation error, bounded by 2e-4 x sum |W x| (K <= 3072 terms, 2^-24 each)
    tol = 2.0 ** -8 * np.abs(exp) + 2e-4 * mag + 1e-30
    bad = np.abs(got - exp) > tol
    assert not bad.any(), f"{where}: {bad.sum()} elements off, worst {np.abs(got - exp)[bad].max():.3g}"


def _project_check(L, seed, lengths, rows_pos, k_off_given=True, q_lora=1536, hidden=3072):
    f = S.bf16_bits_to_f64
    c_q, h, wq_b, wk, wp, g = _project_inputs(seed, len(rows_pos), q_lora, hidden)
    lengths = np.asarray(lengths, dtype=np.int64)
    off = S.offsets(lengths)
    total = int(off[-1])
    cache0 = S.normal_bf16(seed, S.tid(1, S.K_IDX), 0, total * 128).reshape(total, 128)
    k_cache = bf16_dev(cache0)
    n = len(rows_pos)
    seq = np.array([s for s, _ in rows_pos], dtype=np.int32)
    pos = np.array([p for _, p in rows_pos], dtype=np.int32)
    q_out = torch.empty((n, 32, 128), dtype=torch.bfloat16, device="cuda")
    w_out = torch.empty((n, 32), device="cuda")
    cfg = L.LsaConfig()
    ws = L.workspace(cfg, L.OP_INDEX_PROJECT, n, 1, int(lengths.max()))
    L.index_project(cfg, i32_dev(seq) if k_off_given else None, i32_dev(pos), i64_dev(off) if k_off_given else None,
                    int(lengths.max()), bf16_dev(c_q), bf16_dev(h), bf16_dev(wq_b), bf16_dev(wk), bf16_dev(wp),
                    bf16_dev(g), q_out, w_out, k_cache, ws)
    assert L.device_error() == 0
    gq, gw = bf16_host_f64(q_out), w_out.cpu().numpy().astype(np.float64)
    gk = k_cache.view(torch.int16).cpu().numpy().view(np.uint16)
    slots = (off[seq] + pos) if k_off_given else pos.astype(np.int64)
    untouched = np.ones(total, dtype=bool)
    untouched[slots] = False
    np.testing.assert_array_equal(gk[untouched], cache0[untouched])   # only the rows' own slots change
    Wq, Wk, Wp, G = f(wq_b), f(wk), f(wp), f(g)
    for r in range(n):
        cq, hr = f(c_q[r]), f(h[r])
        q, k, w = R.index_project_row(cq, hr, Wq, Wk, Wp, G, int(pos[r]))
        mq = _pair_bound((np.abs(Wq) @ np.abs(cq)).reshape(32, 128))
        raw = Wk @ hr
        scale = np.abs(G) / np.sqrt(np.mean(raw * raw) + 1e-6)
        mk = _pair_bound(scale * (np.abs(Wk) @ np.abs(hr)))
        _check_bf16(gq[r], q, mq, f"q row {r}")
        _check_bf16(f(gk[slots[r]]), k, mk, f"k row {r}")
        assert np.all(np.abs(gw[r] - w) <= 2e-4 * (np.abs(Wp) @ np.abs(hr))), f"w row {r}"


def test_index_project_decode_varlen(L):
    # one new token per sequence, at the last slot of its (already extended) cache
    lengths = [3, 100, 2050, 5000, 777, 100000]
    _project_check(L, 31, lengths, [(b, lengths[b] - 1) for b in range(len(lengths))])


def test_index_project_row_blocks(L):
    # 37 rows over 4 sequences: three 16-row blocks of the fused decode launch, the last ragged
    lengths = [40, 9000, 1, 300]
    rows = [(b, lengths[b] - 1 - i) for b in range(4) for i in range(min(lengths[b], 12))][:37]
    assert len(rows) == 37
    _project_check(L, 33, lengths, rows)


@pytest.mark.parametrize("q_lora,hidden,n", [(512, 1024, 64), (160, 224, 5), (1536, 3072, 65)])
def test_index_project_dims(L, q_lora, hidden, n):
    # fused launch at its row limit; K not a multiple of 512 (tiled GEMMs with split K on
    # few rows); one row past the fused limit
    _project_check(L, 34, [n + 10], [(0, 10 + t) for t in range(n)], q_lora=q_lora, hidden=hidden)


def test_index_project_prefill_rows(L):
    # rows of one sequence at positions 2000 .. 2299 (tiles of 64 rows, a ragged last one)
    _project_check(L, 32, [2300], [(0, 2000 + t) for t in range(300)], k_off_given=False)


# --------------------------------------------------------------------------
# Hierarchical indexing ([LSA-2.0] 分层索引)
# --------------------------------------------------------------------------
def _hier_inputs(seed, lengths, n_rows):
    off = S.offsets(np.asarray(lengths, dtype=np.int64))
    k = S.rms_rows_bf16(seed, S.tid(0, S.K_IDX), 0, int(off[-1]), 128)
    q = S.normal_bf16(seed, S.tid(0, S.Q_IDX), 0, n_rows * 4096).reshape(n_rows, 32, 128)
    w = S.normal_f32(seed, S.tid(0, S.W), 0, n_rows * 32, S.W_SIGMA).reshape(n_rows, 32)
    return off, k, q, w


def _summaries_dev(L, cfg, lengths, k_d, off_d, block):
    blk_off = np.array(L.block_offsets(lengths, block), dtype=np.int64)
    items = [(s, b) for s in range(len(lengths)) for b in range(int(blk_off[s + 1] - blk_off[s]))]
    items = [items[i] for i in np.random.default_rng(1).permutation(len(items))]   # any order
    k_blk = torch.empty((max(int(blk_off[-1]), 1), 128), dtype=torch.bfloat16, device="cuda")
    L.block_summaries(cfg, i32_dev([s for s, _ in items]), i32_dev([b for _, b in items]), k_d, off_d,
                      i64_dev(blk_off), k_blk, block)
    return blk_off, k_blk


def test_block_summaries_bit_exact(L):
    cfg = L.LsaConfig()
    lengths = [1, 63, 64, 65, 1000, 4097]
    off, k, _, _ = _hier_inputs(41, lengths, 1)
    f = S.bf16_bits_to_f64
    for block in (16, 64, 1024):
        blk_off, k_blk = _summaries_dev(L, cfg, lengths, bf16_dev(k), i64_dev(off), block)
        assert L.device_error() == 0
        got = k_blk.view(torch.int16).cpu().numpy().view(np.uint16)
        for s in range(len(lengths)):
            exp = R.block_summaries(f(k[off[s]:off[s + 1]]), block)
            np.testing.assert_array_equal(f(got[blk_off[s]:blk_off[s + 1]]), exp, err_msg=f"block {block} seq {s}")


def test_block_summary_update_after_append(L):
    # decode: after appending a key, re-summarise only the block that holds it
    cfg = L.LsaConfig()
    f = S.bf16_bits_to_f64
    lengths = [130, 64, 1]
    off, k, _, _ = _hier_inputs(42, lengths, 1)
    k_d = bf16_dev(k)
    blk_off = np.array(L.block_offsets([200, 200, 200], 64), dtype=np.int64)   # room to grow
    k_blk = torch.zeros((int(blk_off[-1]), 128), dtype=torch.bfloat16, device="cuda")
    last = [(L_ - 1) // 64 for L_ in lengths]
    L.block_summaries(cfg, i32_dev([0, 1, 2]), i32_dev(last), k_d, i64_dev(off), i64_dev(blk_off), k_blk, 64)
    assert L.device_error() == 0
    got = k_blk.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(3):
        exp = R.block_summaries(f(k[off[s]:off[s + 1]]), 64)[last[s]]
        np.testing.assert_array_equal(f(got[blk_off[s] + last[s]]), exp)


def test_block_summary_bad_item_is_flagged(L):
    cfg = L.LsaConfig()
    off, k, _, _ = _hier_inputs(43, [100], 1)
    blk_off = i64_dev([0, 2])
    k_blk = torch.zeros((2, 128), dtype=torch.bfloat16, device="cuda")
    L.block_summaries(cfg, i32_dev([0]), i32_dev([5]), bf16_dev(k), i64_dev(off), blk_off, k_blk, 64)
    assert L.device_error() == L.DEVERR_POS
    assert not k_blk.view(torch.int16).any()


def _hier_check_row(got_idx, got_cnt, q, w, k_seq, p, ocfg, block, n_blocks, where):
    """Checks one row of a GPU hierarchical selection against the oracle.
    Returns True when the row was compared bit for bit."""
    kb = R.block_summaries(k_seq, block)
    sel, dense, kept = R.hier_select(q, w, k_seq, kb, p, ocfg, block, n_blocks)
    n = p + 1
    if dense:
        assert got_cnt == n, where
        np.testing.assert_array_equal(np.sort(got_idx[:n]), np.arange(n))
        assert np.all(got_idx[n:] == -1)
        return True
    assert got_cnt == ocfg.index_topk, where
    g = got_idx[: ocfg.index_topk]
    assert len(np.unique(g)) == len(g) and g.min() >= 0 and g.max() <= p, where
    forced = set(range(min(ocfg.index_init_tokens, n))) | set(range(max(0, n - ocfg.index_local_tokens), n))
    assert forced <= set(g.tolist()), f"forced token missing {where}"
    # coarse boundary: relative gap between the n_blocks-th and next best unforced block
    bc = R.hier_config(ocfg, block, n_blocks)
    nb = p // block + 1
    b = np.arange(nb)
    mid = (b >= bc.index_init_tokens) & (b < nb - bc.index_local_tokens)
    cs = np.sort(R.score_row(q, w, kb[:nb])[mid])[::-1]
    if len(cs) > n_blocks and abs(cs[n_blocks - 1] - cs[n_blocks]) <= GAP_RTOL * abs(cs[n_blocks - 1]):
        return False            # kept blocks may legitimately differ: validity checked above
    kept_tok = set(np.concatenate([np.arange(x * block, min((x + 1) * block, n)) for x in kept]).tolist())
    assert set(g.tolist()) <= kept_tok, f"token outside the kept blocks {where}"
    s = R.score_row(q, w, k_seq[:n])
    cand = np.array(sorted(kept_tok - forced))
    v = np.sort(s[cand])[::-1]
    k_rem = ocfg.index_topk - len(forced)
    if len(v) <= k_rem or abs(v[k_rem - 1] - v[k_rem]) > GAP_RTOL * abs(v[k_rem - 1]):
        np.testing.assert_array_equal(np.sort(g), sel, err_msg=where)
        return True
    a, e = s[sorted(set(g.tolist()) - forced)].sum(), s[sorted(set(sel.tolist()) - forced)].sum()
    assert abs(a - e) <= GAP_RTOL * abs(e), f"near-tie sum {where}"
    return False


def _hier_run(L, cfg, seed, lengths, rows, block, n_blocks):
    """rows: (sequence, position) pairs. Returns (idx, count, status) and the host inputs."""
    off, k, q, w = _hier_inputs(seed, lengths, len(rows))
    k_d, off_d = bf16_dev(k), i64_dev(off)
    blk_off, k_blk = _summaries_dev(L, cfg, lengths, k_d, off_d, block)
    n = len(rows)
    max_len = int(max(lengths))
    idx = torch.full((n, cfg.index_topk), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    ws = L.hier_workspace(cfg, n, max_len, block, n_blocks)
    st = L.hier_select(cfg, i32_dev([s for s, _ in rows]), i32_dev([p for _, p in rows]), bf16_dev(q), f32_dev(w),
                       k_d, off_d, k_blk, i64_dev(blk_off), max_len, idx, cnt, ws, block, n_blocks)
    assert L.device_error() == 0
    return idx.cpu().numpy(), cnt.cpu().numpy(), st, (off, k, q, w)


def _hier_check(L, cfg, seed, lengths, rows, block, n_blocks, min_exact):
    idx, cnt, _, (off, k, q, w) = _hier_run(L, cfg, seed, lengths, rows, block, n_blocks)
    f = S.bf16_bits_to_f64
    ocfg = oracle_cfg(cfg)
    exact = 0
    for r, (s, p) in enumerate(rows):
        exact += _hier_check_row(idx[r], int(cnt[r]), f(q[r]), w[r].astype(np.float64), f(k[off[s]:off[s + 1]]),
                                 p, ocfg, block, n_blocks, f"row {r} (seq {s}, pos {p})")
    assert exact >= min_exact, f"only {exact} of {len(rows)} rows compared exactly"


def test_hier_select_decode_varlen(L):
    lengths = [3000, 5000, 777, 20000, 2049, 2048, 40000]
    rows = [(s, n - 1) for s, n in enumerate(lengths)]
    _hier_check(L, L.LsaConfig(), 5, lengths, rows, 64, 32, min_exact=5)   # two rows with a near-tie


def test_hier_select_prefill_rows(L):
    # 200 rows of one sequence at consecutive positions (prefill shape)
    rows = [(0, 11800 + t) for t in range(200)]
    # (of the 200 rows, 105 have no near-tie at either stage's boundary in the oracle)
    _hier_check(L, L.LsaConfig(), 6, [12000], rows, 32, 80, min_exact=105)


@pytest.mark.parametrize("block,n_blocks,n_exact", [(16, 256, 3), (128, 16, 2), (1024, 2, 2)])
def test_hier_select_block_sizes(L, block, n_blocks, n_exact):
    # n_exact: rows without a near-tie at either boundary in the oracle
    lengths = [6000, 15000, 2500]
    rows = [(s, n - 1) for s, n in enumerate(lengths)] + [(1, 9000), (1, 100)]
    _hier_check(L, L.LsaConfig(), 7, lengths, rows, block, n_blocks, min_exact=n_exact)


def test_hier_select_tiny_config(L):
    cfg = L.LsaConfig(index_topk=8, index_init_tokens=2, index_local_tokens=4)
    lengths = [40, 100, 300, 5]
    rows = [(s, n - 1) for s, n in enumerate(lengths)] + [(2, 150), (2, 16)]
    _hier_check(L, cfg, 8, lengths, rows, 16, 1, min_exact=6)


def test_hier_every_block_kept_is_the_flat_selection(L):
    # n_blocks covering every block: the GPU's two-stage result equals its flat
    # indexer + top-k on the same inputs, set for set
    cfg = L.LsaConfig()
    lengths = [9000, 30000, 1500]
    rows = [(s, n - 1) for s, n in enumerate(lengths)]
    idx, cnt, _, (off, k, q, w) = _hier_run(L, cfg, 9, lengths, rows, 64, 2048 - 18)
    max_len = int(max(lengths))
    scores = torch.empty((len(rows), max_len), device="cuda")
    L.index_scores(cfg, i32_dev([s for s, _ in rows]), i32_dev([p for _, p in rows]), bf16_dev(q), f32_dev(w),
                   bf16_dev(k), i64_dev(off), max_len, scores)
    fidx = torch.empty((len(rows), cfg.index_topk), dtype=torch.int32, device="cuda")
    fcnt = torch.empty((len(rows),), dtype=torch.int32, device="cuda")
    L.topk(cfg, i32_dev([p for _, p in rows]), max_len, scores, fidx, fcnt,
           L.workspace(cfg, L.OP_TOPK, len(rows), len(rows), max_len))
    fidx, fcnt = fidx.cpu().numpy(), fcnt.cpu().numpy()
    np.testing.assert_array_equal(cnt, fcnt)
    for r in range(len(rows)):
        np.testing.assert_array_equal(np.sort(idx[r, :cnt[r]]), np.sort(fidx[r, :fcnt[r]]))


def test_hier_all_dense_status(L):
    cfg = L.LsaConfig()
    _, cnt, st, _ = _hier_run(L, cfg, 10, [2048, 500], [(0, 2047), (1, 499)], 64, 32)
    assert st == L.LSA_DENSE
    np.testing.assert_array_equal(cnt, [2048, 500])


@pytest.mark.parametrize("name,batch,lo,hi,sample,n_exact", [
    ("decode_b16_128k", 16, 131072, 131072, (0, 9, 13, 14), 3),
    ("decode_b64_16k_32k", 64, 16384, 32768, (5, 40), 0),
])
def test_full_size_hier_sampled(L, name, batch, lo, hi, sample, n_exact):
    # the bench's hierarchical configuration (64-key blocks, 128 kept) at full
    # size; sampled rows re-drawn on the host and checked against the oracle.
    # n_exact: sampled rows with no near-tie at either boundary (128K rows 0, 9,
    # 14); the others are checked by validity, kept blocks and score sums
    from sparse_attention_03_b200.device_inputs import DeviceWorkload
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    block, n_blocks = 64, 128
    lengths = S.decode_lengths(0, batch, lo, hi)
    wl = DeviceWorkload(0, 0, lengths, cli=1, draw_latent=False)
    n = wl.n_rows
    blk_off = np.array(L.block_offsets(lengths, block), dtype=np.int64)
    items = [(s, b) for s in range(n) for b in range(int(blk_off[s + 1] - blk_off[s]))]
    k_blk = torch.empty((int(blk_off[-1]), 128), dtype=torch.bfloat16, device="cuda")
    L.block_summaries(cfg, i32_dev([s for s, _ in items]), i32_dev([b for _, b in items]), wl.k_idx, wl.k_off,
                      i64_dev(blk_off), k_blk, block)
    idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    ws = L.hier_workspace(cfg, n, wl.max_len, block, n_blocks)
    L.hier_select(cfg, wl.seq_of_row, wl.pos, wl.q_idx, wl.w, wl.k_idx, wl.k_off, k_blk, i64_dev(blk_off),
                  wl.max_len, idx, cnt, ws, block, n_blocks)
    assert L.device_error() == 0
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    kb_got = k_blk.view(torch.int16).cpu().numpy().view(np.uint16)
    k_off = S.offsets(lengths)
    f = S.bf16_bits_to_f64
    exact = 0
    for b in sample:
        p = int(lengths[b]) - 1
        a, e = int(k_off[b]), int(k_off[b + 1])
        q = f(S.normal_bf16(0, S.tid(0, S.Q_IDX), b * 4096, 4096)).reshape(32, 128)
        w = S.normal_f32(0, S.tid(0, S.W), b * 32, 32, S.W_SIGMA).astype(np.float64)
        k = f(S.rms_rows_bf16(0, S.tid(0, S.K_IDX), a, e - a, 128))
        np.testing.assert_array_equal(f(kb_got[blk_off[b]:blk_off[b + 1]]), R.block_summaries(k, block),
                                      err_msg=f"{name} row {b} summaries")
        exact += _hier_check_row(idx[b], int(cnt[b]), q, w, k, p, ocfg, block, n_blocks, f"{name} row {b}")
    assert exact >= n_exact
    del wl
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------
# MLA over top-k lists with the forced columns attended first
# --------------------------------------------------------------------------
def _topk_lists(L, cfg, wl, d, max_len):
    n = wl.n_rows
    scores = torch.empty((n, max_len), device="cuda")
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], max_len, scores)
    idx = torch.full((n, cfg.index_topk), -3, dtype=torch.int32, device="cuda")
    cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
    L.topk(cfg, d["pos"], max_len, scores, idx, cnt, L.workspace(cfg, L.OP_TOPK, n, n, max_len))
    return idx, cnt


def test_mla_decode_lists_from_topk(L):
    # dense rows (<= 2048 keys) and selected rows, the lists from the library's top-k
    cfg = L.LsaConfig()
    ocfg = oracle_cfg(cfg)
    lengths = [700, 2048, 2049, 3001, 5000, 9000, 12345, 1]
    wl = S.Workload(11, 2, lengths)
    d = _upload(wl)
    n, max_len = wl.n_rows, max(lengths)
    idx, cnt = _topk_lists(L, cfg, wl, d, max_len)
    ws = L.workspace(cfg, L.OP_MLA_DECODE, n, n, max_len)
    res = {}
    for mode in (False, True):
        out = torch.empty((n, 32, 512), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((n, 32), device="cuda")
        L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], idx, cnt, max_len, out, lse, ws,
                            lists_from_topk=mode)
        assert L.device_error() == 0
        res[mode] = (bf16_host_f64(out), lse.cpu().numpy())
    # the two entry points attend over the same sets in different orders
    assert np.abs(res[True][0] - res[False][0]).max() <= 1e-2
    assert np.abs(res[True][1] - res[False][1]).max() <= 1e-4
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for r in range(n):
        q, w, k, qa, lat = host_rows(wl, r)
        p = int(wl.pos[r])
        s = R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, k.shape[0], ocfg)
        exact = check_selection(idx_h[r], int(cnt_h[r]), s, p, ocfg, where=f"row {r}")
        sel, _ = R.select_topk(s, p, ocfg)
        o, l = R.mla(qa[0], lat[0][sel], ocfg)
        assert_attention(res[True][0][r], res[True][1][r], o, l, check_lse=exact, where=f"row {r}")


def test_mla_decode_topk_bad_count_is_flagged(L):
    cfg = L.LsaConfig()
    lengths = [5000, 3000]
    wl = S.Workload(12, 2, lengths, cli=1)
    d = _upload(wl)
    idx, cnt = _topk_lists(L, cfg, wl, d, max(lengths))
    cnt[1] = 100  # not what the top-k wrote for a row of 3000 keys
    out = torch.empty((2, 32, 512), dtype=torch.bfloat16, device="cuda")
    L.sparse_mla_decode(cfg, d["q_abs"][0], d["latent"][0], d["k_off"], idx, cnt, max(lengths), out, None,
                        L.workspace(cfg, L.OP_MLA_DECODE, 2, 2, max(lengths)), lists_from_topk=True)
    assert L.device_error() == L.DEVERR_COUNT


def test_topk_multi_cta_with_indexer_histogram_twice(L):
    # few long rows (the multi-CTA select): its counters live beside the indexer's
    # histogram and are cleared by the call itself, so a second call on the same
    # histogram gives the same selection, as does the top-k's own first pass
    cfg = L.LsaConfig()
    lengths = [40000, 33000, 17000, 65536]
    wl = S.Workload(15, 0, lengths, cli=1)
    d = _upload(wl)
    n, max_len = wl.n_rows, max(lengths)
    scores = torch.empty((n, max_len), device="cuda")
    hist = L.topk_hist_buffer(n)
    L.index_scores(cfg, d["seq_of_row"], d["pos"], d["q_idx"], d["w"], d["k_idx"], d["k_off"], max_len, scores,
                   topk_hist=hist)
    ws = L.workspace(cfg, L.OP_TOPK, n, n, max_len)
    outs = []
    for h in (hist, hist, None):
        idx = torch.full((n, 2048), -3, dtype=torch.int32, device="cuda")
        cnt = torch.full((n,), -3, dtype=torch.int32, device="cuda")
        L.topk(cfg, d["pos"], max_len, scores, idx, cnt, ws, topk_hist=h)
        outs.append((np.sort(idx.cpu().numpy(), axis=1), cnt.cpu().numpy()))
    for o in outs[1:]:
        np.testing.assert_array_equal(outs[0][0], o[0])
        np.testing.assert_array_equal(outs[0][1], o[1])
    assert np.all(hist.cpu().numpy()[:, 2048:] == 0)
    assert L.device_error() == 0
