"""Helpers shared by the GPU parity tests: host<->device transfer of the host
generator's arrays, the oracle applied to a workload, and the comparison rules
(tolerances) for scores, selections and attention outputs."""
from __future__ import annotations

import numpy as np
import torch

import lsa_synth as S
from oracle import lsa_ref as R

# Tolerances (scores: fp32 accumulation of exact bf16 products; attention: bf16
# I/O with fp32 accumulation).
SCORE_RTOL = 1e-3
ATT_ATOL = 2e-2
ATT_RTOL = 2e-2
LSE_ATOL = 1e-3
GAP_RTOL = 1e-3


def bf16_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def f32_dev(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def i32_dev(x, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int32)).to(device)


def i64_dev(x, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.int64)).to(device)


def bf16_host_f64(t: torch.Tensor) -> np.ndarray:
    """GPU bf16 output -> fp64 numpy (for comparing outputs only)."""
    return t.float().cpu().numpy().astype(np.float64)


def oracle_cfg(cfg) -> R.LsaConfig:
    return R.LsaConfig(index_topk=cfg.index_topk, index_init_tokens=cfg.index_init_tokens,
                       index_local_tokens=cfg.index_local_tokens, cli_factor=cfg.cli_factor)


def host_rows(wl: S.Workload, r: int):
    """fp64 inputs of row r of a host-drawn workload: q, w, k_seq, [q_abs], [latent_seq]."""
    b = int(wl.seq_of_row[r])
    a, e = int(wl.k_off[b]), int(wl.k_off[b + 1])
    f = S.bf16_bits_to_f64
    return (f(wl.q_idx[r]), wl.w[r].astype(np.float64), f(wl.k_idx[a:e]),
            [f(q[r]) for q in wl.q_abs], [f(c[a:e]) for c in wl.latent])


def score_scale(q, w, k):
    """sum_h |w_h| ReLU(q_h . k): the magnitude the score tolerance is relative to."""
    return np.abs(w) @ np.maximum(q @ k.T, 0.0)


def assert_scores(got_row: np.ndarray, q, w, k, p, cfg: R.LsaConfig, where=""):
    n = p + 1  # columns after p are masked and never written
    exp = R.mask_and_force(R.score_row(q, w, k[:n]), p, n, cfg)
    got_row = got_row[:n]
    fin = np.isfinite(exp)
    assert np.array_equal(np.isposinf(got_row), np.isposinf(exp)), f"forced columns differ {where}"
    assert np.isfinite(got_row[fin]).all(), f"non-finite score {where}"
    tol = SCORE_RTOL * (score_scale(q, w, k[:n])[fin] + 1e-6)
    err = np.abs(got_row[fin] - exp[fin])
    assert np.all(err <= tol), f"scores {where}: max err {err.max()} (tol {tol[err.argmax()]})"


def rank_gap(s_row: np.ndarray, p: int, cfg: R.LsaConfig) -> float:
    """Relative gap between the k-th and (k+1)-th visible scores (the oracle's)."""
    vis = np.sort(s_row[: p + 1])[::-1]
    fin = vis[np.isfinite(vis)]
    k_rem = cfg.index_topk - cfg.index_init_tokens - cfg.index_local_tokens
    a, b = fin[k_rem - 1], fin[k_rem]
    return abs(a - b) / max(abs(a), 1e-30)


def check_selection(got_idx: np.ndarray, got_cnt: int, s_oracle: np.ndarray, p: int,
                    cfg: R.LsaConfig, where="") -> bool:
    """Checks a GPU selection against the oracle's. Returns True when the row's
    set must be (and is) bit-exact, False when a near-tie allowed a score-sum match."""
    n = p + 1
    exp, dense = R.select_topk(s_oracle, p, cfg)
    if dense:
        assert got_cnt == n, f"dense count {where}"
        np.testing.assert_array_equal(np.sort(got_idx[:n]), np.arange(n))
        assert np.all(got_idx[n:] == -1)
        return True
    assert got_cnt == cfg.index_topk, f"count {where}"
    sel = got_idx[: cfg.index_topk]
    assert len(np.unique(sel)) == len(sel), f"duplicates {where}"
    assert sel.min() >= 0 and sel.max() <= p, f"invisible index {where}"
    forced = set(range(min(cfg.index_init_tokens, n))) | set(range(n - cfg.index_local_tokens, n))
    assert forced <= set(sel.tolist()), f"forced column missing {where}"
    if rank_gap(s_oracle, p, cfg) > GAP_RTOL:
        np.testing.assert_array_equal(np.sort(sel), exp, err_msg=f"selection {where}")
        return True
    mid_got = np.array(sorted(set(sel.tolist()) - forced))
    mid_exp = np.array(sorted(set(exp.tolist()) - forced))
    a, b = s_oracle[mid_got].sum(), s_oracle[mid_exp].sum()
    assert abs(a - b) <= GAP_RTOL * abs(b), f"near-tie selection sum {where}: {a} vs {b}"
    return False


def assert_attention(o_got, lse_got, o_exp, lse_exp, check_lse=True, where=""):
    err = np.abs(o_got - o_exp)
    tol = ATT_ATOL + ATT_RTOL * np.abs(o_exp)
    assert np.all(err <= tol), f"attention {where}: max err {err.max()}"
    if check_lse and lse_got is not None:
        lerr = np.abs(lse_got - lse_exp)
        assert np.all(lerr <= LSE_ATOL), f"lse {where}: max err {lerr.max()}"
