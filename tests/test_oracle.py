"""Pins for the fp64 oracle (CPU only).

Each test ties one oracle function to something other than itself: a closed
form, an identity of the mathematics, a brute-force enumeration, or an
independent library routine (torch's scaled_dot_product_attention). A
plausible slip in the oracle (dropped ReLU, wrong head index, sign error,
off-by-one in the window, wrong scale, values taken from the wrong dims) fails
at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import lsa_ref as R
from oracle.lsa_ref import PAGES, TINY, LsaConfig

rng = np.random.default_rng(1234)


# --------------------------------------------------------------------------
# Index scores
# --------------------------------------------------------------------------
def test_score_closed_form_one_head():
    # One head, w = 1, q = e0, keys c * e0: s = ReLU(c).
    c = np.array([-2.0, -0.5, 0.0, 0.25, 3.0])
    q = np.zeros((1, 8)); q[0, 0] = 1.0
    k = np.zeros((5, 8)); k[:, 0] = c
    np.testing.assert_array_equal(R.score_row(q, np.array([1.0]), k), np.maximum(c, 0))
    # negative weight flips the sign of the ReLU'd value
    np.testing.assert_array_equal(R.score_row(q, np.array([-2.0]), k), -2.0 * np.maximum(c, 0))


def test_score_heads_weighted_independently():
    # Two heads looking at different coordinates with different weights.
    q = np.zeros((2, 4)); q[0, 0] = 1.0; q[1, 1] = 1.0
    k = np.array([[1.0, -1.0, 0, 0], [-3.0, 2.0, 0, 0], [0.5, 0.5, 0, 0]])
    w = np.array([0.25, 4.0])
    expect = np.array([0.25 * 1.0 + 0.0, 0.0 + 4.0 * 2.0, 0.25 * 0.5 + 4.0 * 0.5])
    np.testing.assert_allclose(R.score_row(q, w, k), expect, rtol=0, atol=1e-15)


def test_score_odd_part_is_linear():
    # ReLU(x) - ReLU(-x) = x, so s(q) - s(-q) = (sum_h w_h q_h) . k, a plain matmul.
    q = rng.standard_normal((32, 128)); w = rng.standard_normal(32); k = rng.standard_normal((300, 128))
    lhs = R.score_row(q, w, k) - R.score_row(-q, w, k)
    rhs = k @ (w @ q)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-10)


def test_score_even_part_is_weighted_abs():
    # ReLU(x) + ReLU(-x) = |x|.
    q = rng.standard_normal((32, 128)); w = rng.standard_normal(32); k = rng.standard_normal((200, 128))
    lhs = R.score_row(q, w, k) + R.score_row(-q, w, k)
    rhs = np.abs(k @ q.T) @ w
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-10)


def test_score_homogeneity():
    q = rng.standard_normal((32, 128)); w = rng.standard_normal(32); k = rng.standard_normal((64, 128))
    s = R.score_row(q, w, k)
    np.testing.assert_allclose(R.score_row(3.0 * q, w, k), 3.0 * s, rtol=1e-12, atol=1e-10)
    np.testing.assert_allclose(R.score_row(q, -0.5 * w, k), -0.5 * s, rtol=1e-12, atol=1e-10)


# --------------------------------------------------------------------------
# Mask and forcing
# --------------------------------------------------------------------------
@pytest.mark.parametrize("p", [0, 5, 15, 16, 1039, 1040, 2047, 2048, 5000])
def test_mask_and_force_pages_constants(p):
    L = p + 7
    s = mask_and_force_input = np.arange(p + 1, dtype=np.float64)
    out = R.mask_and_force(s, p, L, PAGES)
    assert np.all(np.isneginf(out[p + 1:]))
    forced = set(range(min(16, p + 1))) | set(range(max(0, p + 1 - 1024), p + 1))
    got = set(np.flatnonzero(np.isposinf(out)).tolist())
    assert got == forced
    rest = sorted(set(range(p + 1)) - forced)
    np.testing.assert_array_equal(out[rest], mask_and_force_input[rest])


def test_mask_and_force_tiny():
    out = R.mask_and_force(np.arange(10.0), 9, 12, TINY)
    # sink {0,1}, local {6,7,8,9}, masked {10,11}
    assert np.isposinf(out[[0, 1, 6, 7, 8, 9]]).all()
    np.testing.assert_array_equal(out[2:6], [2.0, 3.0, 4.0, 5.0])
    assert np.isneginf(out[10:]).all()


# --------------------------------------------------------------------------
# Top-k
# --------------------------------------------------------------------------
def _brute_force_topk(s, n, k):
    """The unique k-subset S of 0..n-1 such that every chosen i beats every
    unchosen j: s_i > s_j, or s_i == s_j and i < j. Found by enumeration."""
    found = []
    for sub in itertools.combinations(range(n), k):
        chosen = set(sub)
        ok = all((s[i] > s[j]) or (s[i] == s[j] and i < j)
                 for i in chosen for j in range(n) if j not in chosen)
        if ok:
            found.append(sub)
    assert len(found) == 1
    return np.array(found[0])


@pytest.mark.parametrize("trial", range(12))
def test_topk_brute_force_tiny(trial):
    r = np.random.default_rng(100 + trial)
    n = int(r.integers(9, 13))
    p = n - 1
    # coarse values so that exact ties occur
    s = r.integers(-3, 4, size=n).astype(np.float64)
    row = R.mask_and_force(s, p, n + 3, TINY)
    sel, dense = R.select_topk(row, p, TINY)
    assert not dense
    np.testing.assert_array_equal(sel, _brute_force_topk(row, n, TINY.index_topk))


def test_topk_dense_fallback_boundary():
    for n in (1, 7, 8):
        sel, dense = R.select_topk(np.zeros(n + 2), n - 1, TINY)
        assert dense and np.array_equal(sel, np.arange(n))
    sel, dense = R.select_topk(np.zeros(12), 8, TINY)
    assert not dense and len(sel) == 8


def test_topk_planted_pages_constants():
    # 1008 planted middle columns with the largest finite scores are chosen
    # together with the 16 + 1024 forced columns.
    p = 6000
    r = np.random.default_rng(7)
    s = r.uniform(-1.0, 1.0, p + 1)
    middle = np.arange(16, p + 1 - 1024)
    planted = np.sort(r.choice(middle, 1008, replace=False))
    s[planted] = 10.0 + r.uniform(0, 1, 1008)
    row = R.mask_and_force(s, p, p + 100, PAGES)
    sel, dense = R.select_topk(row, p, PAGES)
    expect = np.sort(np.concatenate([np.arange(16), planted, np.arange(p + 1 - 1024, p + 1)]))
    assert not dense
    np.testing.assert_array_equal(sel, expect)


def test_topk_all_equal_takes_lowest_indices():
    p = 4000
    row = R.mask_and_force(np.zeros(p + 1), p, p + 1, PAGES)
    sel, _ = R.select_topk(row, p, PAGES)
    expect = np.concatenate([np.arange(16), np.arange(16, 16 + 1008), np.arange(p + 1 - 1024, p + 1)])
    np.testing.assert_array_equal(sel, np.sort(expect))


def test_topk_through_scores_planted():
    # Plant through the indexer itself: keys aligned with every head's query
    # score high, keys anti-aligned score 0 (all weights positive).
    p, d = 3500, 128
    r = np.random.default_rng(3)
    u = r.standard_normal(d); u /= np.linalg.norm(u)
    q = np.tile(u, (32, 1)) + 0.01 * r.standard_normal((32, d))
    w = np.abs(r.standard_normal(32)) + 0.1
    k = -np.abs(r.standard_normal((p + 1, 1))) * u + 0.001 * r.standard_normal((p + 1, d))
    planted = np.sort(r.choice(np.arange(16, p + 1 - 1024), 1008, replace=False))
    k[planted] = (5.0 + r.uniform(0, 1, (1008, 1))) * u
    s = R.mask_and_force(R.score_row(q, w, k), p, p + 1, PAGES)
    sel, _ = R.select_topk(s, p, PAGES)
    expect = np.sort(np.concatenate([np.arange(16), planted, np.arange(p + 1 - 1024, p + 1)]))
    np.testing.assert_array_equal(sel, expect)


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------
def test_softmax_scale_from_dims():
    assert PAGES.softmax_scale == pytest.approx(1.0 / math.sqrt(192.0), rel=0, abs=1e-16)


def test_mla_zero_query_is_mean_of_values():
    c = rng.standard_normal((37, 576))
    o, lse = R.mla(np.zeros((32, 576)), c, PAGES)
    np.testing.assert_allclose(o, np.tile(c[:, :512].mean(axis=0), (32, 1)), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, np.full(32, math.log(37)), rtol=1e-14)


def test_mla_single_key():
    c = rng.standard_normal((1, 576)); q = rng.standard_normal((32, 576))
    o, lse = R.mla(q, c, PAGES)
    np.testing.assert_allclose(o, np.tile(c[0, :512], (32, 1)), rtol=1e-14)
    np.testing.assert_allclose(lse, PAGES.softmax_scale * (q @ c[0]), rtol=1e-13)


def test_mla_two_keys_sigmoid():
    c = rng.standard_normal((2, 576)); q = rng.standard_normal((32, 576))
    o, _ = R.mla(q, c, PAGES)
    d = PAGES.softmax_scale * (q @ (c[0] - c[1]))
    a = 1.0 / (1.0 + np.exp(-d))
    np.testing.assert_allclose(o, a[:, None] * c[0, :512] + (1 - a[:, None]) * c[1, :512], rtol=1e-12, atol=1e-13)


def test_mla_one_hot_values_reveal_selection():
    # q = 0 and V[i] = e_{i mod 512}: the output shows exactly which rows were used.
    n = 700
    c = np.zeros((n, 576))
    c[np.arange(n), np.arange(n) % 512] = 1.0
    sel = np.sort(rng.choice(n, 300, replace=False))
    o, _ = R.mla(np.zeros((4, 576)), c[sel], PAGES)
    expect = np.zeros(512)
    np.add.at(expect, sel % 512, 1.0 / 300)
    np.testing.assert_allclose(o[0], expect, atol=1e-15)


def test_mla_matches_torch_sdpa():
    q = rng.standard_normal((32, 576)); c = rng.standard_normal((513, 576))
    o, lse = R.mla(q, c, PAGES)
    tq = torch.from_numpy(q)[None, :, None, :]
    tk = torch.from_numpy(c)[None, None].expand(1, 32, -1, -1)
    tv = torch.from_numpy(c[:, :512])[None, None].expand(1, 32, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=PAGES.softmax_scale)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-12)
    ref_lse = torch.logsumexp(PAGES.softmax_scale * (torch.from_numpy(q) @ torch.from_numpy(c).T), dim=1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-13)


def test_absorbed_equals_explicit_mla():
    # The pages' absorbed-attention test: embed_q / unembed_out == explicit heads.
    H, n = 4, 50
    q_nope = rng.standard_normal((H, 128)); q_rope = rng.standard_normal((H, 64))
    c_kv = rng.standard_normal((n, 512)); k_rope = rng.standard_normal((n, 64))
    w_uk = rng.standard_normal((H, 128, 512)) / 20; w_uv = rng.standard_normal((H, 128, 512)) / 20
    q_abs = R.absorb_query(q_nope, q_rope, w_uk)
    o_lat, _ = R.mla(q_abs, np.concatenate([c_kv, k_rope], axis=1), PAGES)
    absorbed = R.unembed_out(o_lat, w_uv)
    explicit = R.explicit_mla(q_nope, q_rope, c_kv, k_rope, w_uk, w_uv, PAGES)
    np.testing.assert_allclose(absorbed, explicit, rtol=1e-10, atol=1e-12)
    # and the explicit heads against torch's attention on the explicit tensors
    for h in range(H):
        k = np.concatenate([c_kv @ w_uk[h].T, k_rope], axis=1)
        v = c_kv @ w_uv[h].T
        qq = np.concatenate([q_nope[h], q_rope[h]])
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qq)[None, None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
            scale=PAGES.softmax_scale)
        np.testing.assert_allclose(explicit[h], ref[0, 0].numpy(), rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# Whole row: invariants from the pages
# --------------------------------------------------------------------------
def _row_inputs(L, d_idx=128, seed=0):
    r = np.random.default_rng(seed)
    return (r.standard_normal((32, d_idx)), r.standard_normal(32) / math.sqrt(32),
            r.standard_normal((L, d_idx)), [r.standard_normal((32, 576)) for _ in range(2)],
            [r.standard_normal((L, 576)) for _ in range(2)])


def test_dense_fallback_equals_dense_mla():
    # (a) cached length <= 2048: the result is dense MLA.
    q, w, k, qa, lat = _row_inputs(2048)
    sel, dense, outs = R.lsa_row(q, w, k, 2047, qa, lat, PAGES)
    assert dense and len(sel) == 2048
    for z in range(2):
        o, lse = R.dense_mla_row(qa[z], lat[z], 2047)
        np.testing.assert_array_equal(outs[z][0], o)


def test_topk_at_least_length_equals_dense():
    # (b) topk >= cached length in a generic config: sparse == dense.
    cfg = LsaConfig(index_topk=64, index_init_tokens=2, index_local_tokens=4)
    q, w, k, qa, lat = _row_inputs(60)
    _, dense, outs = R.lsa_row(q, w, k, 59, qa, lat, cfg)
    assert dense
    # force the sparse branch with topk == n explicitly
    s = R.mask_and_force(R.score_row(q, w, k), 59, 60, cfg)
    sel = np.argsort(-s, kind="stable")[:60]
    o, _ = R.mla(qa[0], lat[0][np.sort(sel)], cfg)
    np.testing.assert_allclose(outs[0][0], o, rtol=1e-13, atol=1e-13)


def test_sink_and_local_always_selected():
    # (c) even when their scores are the lowest possible.
    p = 3000
    q, w, k, qa, lat = _row_inputs(p + 1, seed=5)
    w = np.abs(w)
    k[:16] = -10 * q.mean(axis=0)               # sinks score ~0
    k[p + 1 - 1024:] = -10 * q.mean(axis=0)      # local window scores ~0
    sel, dense, _ = R.lsa_row(q, w, k, p, qa, lat, PAGES)
    assert not dense and len(sel) == 2048
    assert set(range(16)) <= set(sel.tolist())
    assert set(range(p + 1 - 1024, p + 1)) <= set(sel.tolist())


def test_cli_sharing_equals_two_passes():
    # (e) two sub-blocks sharing one index pass == two passes on the same indices.
    p = 2600
    q, w, k, qa, lat = _row_inputs(p + 1, seed=9)
    sel, _, outs = R.lsa_row(q, w, k, p, qa, lat, PAGES)
    for z in range(2):
        sel_z, _, outs_z = R.lsa_row(q, w, k, p, [qa[z]], [lat[z]], PAGES)
        np.testing.assert_array_equal(sel_z, sel)
        np.testing.assert_array_equal(outs_z[0][0], outs[z][0])


def test_decode_equals_prefill_row():
    # Cached decode at length p+1 equals row p of a prefill over the same cache.
    L = 2300
    q, w, k, qa, lat = _row_inputs(L, seed=11)
    for p in (100, 2047, 2048, 2299):
        sel_d, _, outs_d = R.lsa_row(q, w, k[: p + 1], p, qa, [x[: p + 1] for x in lat], PAGES)
        sel_p, _, outs_p = R.lsa_row(q, w, k, p, qa, lat, PAGES)
        np.testing.assert_array_equal(sel_d, sel_p)
        np.testing.assert_array_equal(outs_d[1][0], outs_p[1][0])


def test_tiny_config_whole_row():
    # The pages' tiny LSA config (topk 8, init 2, local 4) end to end.
    L = 20
    q, w, k, qa, lat = _row_inputs(L, seed=13)
    for p in range(L):
        sel, dense, outs = R.lsa_row(q, w, k, p, qa, lat, TINY)
        n = p + 1
        assert dense == (n <= 8)
        assert len(sel) == min(n, 8) and len(set(sel.tolist())) == len(sel)
        assert sel.max() <= p
        if not dense:
            assert {0, 1, p - 3, p - 2, p - 1, p} <= set(sel.tolist())
        assert np.isfinite(outs[0][0]).all()


# --------------------------------------------------------------------------
# MTP draft round: the draft steps share one index pass
# ([LSA-2.0] 多token预测模块集成)
# --------------------------------------------------------------------------
def _tagged_latent(L):
    # V[j] = e_j: with q = 0 the output is the mean of the attended keys' tags
    c = np.zeros((L, 576))
    c[np.arange(L), np.arange(L)] = 1.0
    return c


def test_mtp_round_hand_worked_tiny():
    # Tiny config (topk 8, init 2, local 4), 15 cached keys, first draft step at
    # p = 11 (12 visible keys > 8: sparse). One index head with weight 1 and
    # q = e_0 makes score_j = max(k[j, 0], 0). Worked by hand: the forced columns
    # are the sinks {0, 1} and the local window {8, 9, 10, 11}; of the middle
    # columns 2..7 the two best are 3 (5.0) and 6 (4.0). Step 0 attends over
    # that set; step 1 (query at 12) adds key 12; step 2 (query at 13) adds 12
    # and 13. Key 14 is never attended (no draft has reached it).
    L, p = 15, 11
    q = np.zeros((32, 128)); q[0, 0] = 1.0
    w = np.zeros(32); w[0] = 1.0
    k = np.zeros((L, 128))
    k[:, 0] = [0.1, 0.2, 0.3, 5.0, 0.5, 0.6, 4.0, 0.7, 9.0, 9.0, 9.0, 9.0, 9.0, 9.0, 9.0]
    lat = _tagged_latent(L)
    sel, dense, outs = R.mtp_round(q, w, k, p, [np.zeros((32, 576))] * 3, lat, TINY)
    assert not dense
    np.testing.assert_array_equal(sel, [0, 1, 3, 6, 8, 9, 10, 11])
    sets = [[0, 1, 3, 6, 8, 9, 10, 11], [0, 1, 3, 6, 8, 9, 10, 11, 12], [0, 1, 3, 6, 8, 9, 10, 11, 12, 13]]
    for i, keys in enumerate(sets):
        expect = np.zeros(512)
        expect[keys] = 1.0 / len(keys)
        np.testing.assert_allclose(outs[i][0], np.tile(expect, (32, 1)), atol=1e-15)
        np.testing.assert_allclose(outs[i][1], np.full(32, math.log(len(keys))), rtol=1e-14)


def test_mtp_round_dense_steps_are_dense_attention():
    # p + 1 <= topk: no selection; step i is plain softmax attention over keys
    # 0 .. p+i, checked against torch's attention on those keys.
    L, p = 140, 100
    r = np.random.default_rng(3)
    q, w, k = r.standard_normal((32, 128)), r.standard_normal(32), r.standard_normal((L, 128))
    qs = [r.standard_normal((32, 576)) for _ in range(3)]
    lat = r.standard_normal((L, 576))
    sel, dense, outs = R.mtp_round(q, w, k, p, qs, lat, PAGES)
    assert dense and np.array_equal(sel, np.arange(p + 1))
    for i in range(3):
        c = lat[: p + 1 + i]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qs[i])[None, :, None, :], torch.from_numpy(c)[None, None].expand(1, 32, -1, -1),
            torch.from_numpy(c[:, :512])[None, None].expand(1, 32, -1, -1), scale=PAGES.softmax_scale)
        np.testing.assert_allclose(outs[i][0], ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-12)


def test_mtp_round_shares_the_first_steps_selection():
    # pages' constants, sparse: every step reuses step 0's selection (made at p,
    # forced window p-1023 .. p) and adds only its new keys; step 0 is the
    # layer path's sub-block. A step that ran its own index pass would drop
    # p-1023 .. p-1023+i from its window; one that skipped its new keys would
    # miss p+1 .. p+i: the tagged values show both.
    p, L = 3000, 3003
    r = np.random.default_rng(4)
    q, w, k = r.standard_normal((32, 128)), r.standard_normal(32) / math.sqrt(32), r.standard_normal((L, 128))
    lat = np.zeros((L, 576))
    lat[np.arange(L), np.arange(L) % 512] = 1.0
    sel, dense, outs = R.mtp_round(q, w, k, p, [np.zeros((32, 576))] * 3, lat, PAGES)
    sel0, _, outs0 = R.lsa_row(q, w, k[: p + 1], p, [np.zeros((32, 576))], [lat[: p + 1]], PAGES)
    np.testing.assert_array_equal(sel, sel0)
    np.testing.assert_array_equal(outs[0][0], outs0[0][0])
    assert not dense and {p - 1023, p} <= set(sel.tolist()) and sel.max() == p
    for i in range(3):
        keys = np.concatenate([sel, np.arange(p + 1, p + 1 + i)])
        expect = np.zeros(512)
        np.add.at(expect, keys % 512, 1.0 / len(keys))
        np.testing.assert_allclose(outs[i][0][0], expect, atol=1e-15)


# --------------------------------------------------------------------------
# Indexer projection (upstream of the path): RoPE, RMSNorm, the projections.
# --------------------------------------------------------------------------
def test_rope_closed_form_frequencies():
    # pair i of the rope part turns by pos * theta^(-2i/64): a unit vector on the
    # pair's first dim lands on (cos, sin) of exactly that angle
    pos = 777
    for i in (0, 1, 17, 31):
        x = np.zeros(128)
        x[64 + i] = 1.0
        y = R.rope(x, pos)
        ang = pos * R.ROPE_THETA ** (-2.0 * i / 64)
        assert abs(y[64 + i] - np.cos(ang)) < 1e-12 and abs(y[96 + i] - np.sin(ang)) < 1e-12
        assert np.count_nonzero(np.abs(y) > 1e-15) <= 2


def test_rope_relative_position_and_norms():
    # dot products of rotated vectors depend only on the position difference;
    # a sign slip in one half of the rotation breaks this; norms of pairs are kept
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((2, 128))
    for p1, p2 in ((10, 3), (983039, 5), (1, 1)):
        lhs = R.rope(q, p1)[64:] @ R.rope(k, p2)[64:]
        rhs = R.rope(q, p1 - p2)[64:] @ k[64:]
        assert abs(lhs - rhs) < 1e-9 * (1 + abs(rhs))
    y = R.rope(q, 12345)
    np.testing.assert_array_equal(y[:64], q[:64])          # the non-rope half is untouched
    np.testing.assert_allclose(y[64:96] ** 2 + y[96:] ** 2, q[64:96] ** 2 + q[96:] ** 2, rtol=1e-12)


def test_rms_norm_closed_form():
    w = np.linspace(0.5, 1.5, 128)
    for c in (3.0, -0.25):
        y = R.rms_norm(np.full(128, c), w)
        np.testing.assert_allclose(y, np.sign(c) * abs(c) / np.sqrt(c * c + R.NORM_EPS) * w, rtol=1e-13)
    x = np.zeros(128)
    x[0], x[1] = 3.0, 4.0            # mean square 25/128
    np.testing.assert_allclose(R.rms_norm(x, np.ones(128))[:2], np.array([3.0, 4.0]) / np.sqrt(25 / 128 + 1e-6),
                               rtol=1e-13)


def test_index_project_layout_and_pieces():
    # head-major query rows, the key normalised before it is rotated, raw weights
    rng = np.random.default_rng(6)
    K = 16
    c_q, h = rng.standard_normal(K), rng.standard_normal(K)
    wq_b, wk, wp = rng.standard_normal((4096, K)), rng.standard_normal((128, K)), rng.standard_normal((32, K))
    g = rng.uniform(0.5, 1.5, 128)
    q, k, w = R.index_project_row(c_q, h, wq_b, wk, wp, g, pos=0)
    for head in (0, 13, 31):
        np.testing.assert_allclose(q[head], wq_b[128 * head:128 * (head + 1)] @ c_q, rtol=1e-12)
    raw = wk @ h
    np.testing.assert_allclose(k, raw / np.sqrt(np.mean(raw * raw) + 1e-6) * g, rtol=1e-12)
    np.testing.assert_allclose(w, wp @ h, rtol=1e-12)
    q5, k5, _ = R.index_project_row(c_q, h, wq_b, wk, wp, g, pos=5)
    np.testing.assert_allclose(q5, R.rope(q, 5), rtol=1e-12)
    np.testing.assert_allclose(k5, R.rope(k, 5), rtol=1e-12)


# ---------------------------------------------------------------------------
# Hierarchical indexing ([LSA-2.0] 分层索引)
# ---------------------------------------------------------------------------
def test_bf16_round_ties_and_halfway():
    one = 1.0
    ulp = 2.0 ** -7
    cases = {
        one + ulp / 2: one,                        # tie -> even (1.0)
        one + 3 * ulp / 2: one + 2 * ulp,          # tie -> even (1 + 2 ulp)
        one + ulp / 2 + 2.0 ** -40: one + ulp,     # just above the tie rounds up
        one + ulp / 2 - 2.0 ** -40: one,           # just below rounds down
        -(one + 3 * ulp / 2): -(one + 2 * ulp),
        255.5: 256.0,                              # 8 significant bits: 255.5 is a tie, 256 is even
        3.0 * 2.0 ** -100: 3.0 * 2.0 ** -100,      # already representable
    }
    got = R.bf16_round(np.array(list(cases)))
    np.testing.assert_array_equal(got, np.array(list(cases.values())))


def test_bf16_round_matches_torch_on_fp32_values():
    # inputs exactly representable in fp32, where torch's conversion rounds once
    x = np.random.default_rng(3).standard_normal(20000).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(R.bf16_round(x), ref)


def test_block_summaries_closed_forms():
    k = np.zeros((10, 3))
    k[0:4] = [1.0, 2.0, -3.0]                      # a block of identical keys -> that key
    k[4:8] = [[0, 0, 1], [0, 0, 3], [1, 1, 5], [3, 1, 7]]   # mean (1, 0.5, 4)
    k[8:10] = [[2, 4, 8], [4, 8, 16]]              # short last block: mean of its 2 keys
    s = R.block_summaries(k, 4)
    np.testing.assert_array_equal(s, [[1, 2, -3], [1, 0.5, 4], [3, 6, 12]])


def test_hier_config_forced_blocks_cover_forced_tokens():
    # every forced token lies in a forced block, for every alignment of p
    for cfg, block in ((TINY, 4), (TINY, 2), (PAGES, 64), (PAGES, 16), (PAGES, 128)):
        bcfg = R.hier_config(cfg, block, 4)
        for p in range(0, 4 * cfg.index_local_tokens + 3 * block, max(1, block // 3)):
            pb = p // block
            j = np.arange(p + 1)
            forced = j[(j < cfg.index_init_tokens) | (j >= p + 1 - cfg.index_local_tokens)]
            b = np.arange(pb + 1)
            fb = set(b[(b < bcfg.index_init_tokens) | (b >= pb + 1 - bcfg.index_local_tokens)].tolist())
            assert set((forced // block).tolist()) <= fb, (cfg, block, p)


def _rand_case(rng, L, d=8, heads=4):
    q = rng.standard_normal((heads, d))
    w = rng.standard_normal(heads)
    k = R.bf16_round(rng.standard_normal((L, d)))
    return q, w, k


@pytest.mark.parametrize("trial", range(6))
def test_hier_with_every_block_kept_is_flat_lsa(trial):
    # n_blocks at least the number of blocks: the coarse stage keeps everything and
    # the result is the flat selection
    rng = np.random.default_rng(100 + trial)
    L, block = 300, 8
    q, w, k = _rand_case(rng, L)
    kb = R.block_summaries(k, block)
    for p in (3, 7, 8, 9, 100, 299):
        sel, dense, kept = R.hier_select(q, w, k, kb, p, TINY, block, n_blocks=L)
        np.testing.assert_array_equal(kept, np.arange(p // block + 1))
        flat, fdense = R.select_topk(R.mask_and_force(R.score_row(q, w, k[: p + 1]), p, L, TINY), p, TINY)
        assert dense == fdense
        np.testing.assert_array_equal(sel, flat)


def _brute_hier(q, w, k, p, cfg, block, n_blocks):
    # independent restatement with explicit loops and tuple sorts
    nb = p // block + 1
    n_init = math.ceil(cfg.index_init_tokens / block)
    n_loc = math.ceil(cfg.index_local_tokens / block) + 1
    def score(key):
        return sum(w[h] * max(float(np.dot(q[h], key)), 0.0) for h in range(len(w)))
    means = []
    for b in range(nb):
        rows = k[b * block: min((b + 1) * block, len(k))]
        means.append(R.bf16_round(sum(rows) / len(rows)))
    if nb <= n_init + n_loc + n_blocks:
        kept = list(range(nb))
    else:
        forced = [b for b in range(nb) if b < n_init or b >= nb - n_loc]
        rest = sorted((b for b in range(nb) if b not in forced), key=lambda b: (-score(means[b]), b))
        kept = sorted(forced + rest[:n_blocks])
    if p + 1 <= cfg.index_topk:
        return list(range(p + 1)), kept
    cand = [j for b in kept for j in range(b * block, min((b + 1) * block, p + 1))]
    def key(j):
        forced = j < cfg.index_init_tokens or j >= p + 1 - cfg.index_local_tokens
        return (0 if forced else 1, -score(k[j]) if not forced else 0.0, j)
    return sorted(sorted(cand, key=key)[: cfg.index_topk]), kept


@pytest.mark.parametrize("trial", range(10))
def test_hier_brute_force_tiny(trial):
    rng = np.random.default_rng(200 + trial)
    L, block, nbk = 90, 4, 3
    q, w, k = _rand_case(rng, L)
    kb = R.block_summaries(k, block)
    for p in (5, 9, 20, 47, 60, 89):
        sel, dense, kept = R.hier_select(q, w, k, kb, p, TINY, block, nbk)
        bsel, bkept = _brute_hier(q, w, k, p, TINY, block, nbk)
        np.testing.assert_array_equal(kept, bkept)
        np.testing.assert_array_equal(sel, bsel)


def test_hier_planted_blocks_survive():
    # keys of blocks 10 and 20 point along the query; everything else is orthogonal
    rng = np.random.default_rng(7)
    L, block, d = 2000, 16, 8
    q = np.zeros((2, d)); q[:, 0] = 1.0
    w = np.array([1.0, 0.5])
    k = np.zeros((L, d)); k[:, 1:] = R.bf16_round(rng.standard_normal((L, d - 1)))
    k[10 * block:11 * block, 0] = 2.0
    k[20 * block:21 * block, 0] = 1.0
    kb = R.block_summaries(k, block)
    cfg = LsaConfig(index_topk=24, index_init_tokens=2, index_local_tokens=4)
    sel, dense, kept = R.hier_select(q, w, k, kb, L - 1, cfg, block, n_blocks=2)
    # sink block 0, the ceil(4/16)+1 = 2 most recent blocks, and the planted two
    np.testing.assert_array_equal(kept, [0, 10, 20, 123, 124])
    # forced tokens (0, 1, and the last 4) plus the 16 keys of block 10 and the
    # lowest-index 2 of block 20 (all its keys tie)
    expect = sorted([0, 1, *range(L - 4, L), *range(160, 176), 320, 321])
    np.testing.assert_array_equal(sel, expect)
    assert not dense


def test_hier_kept_sets_nest_with_n_blocks():
    rng = np.random.default_rng(11)
    L, block = 3000, 16
    q, w, k = _rand_case(rng, L)
    kb = R.block_summaries(k, block)
    prev = None
    for nbk in (1, 2, 5, 10, 40, 200):
        _, _, kept = R.hier_select(q, w, k, kb, L - 1, PAGES, block, nbk)
        if prev is not None:
            assert set(prev) <= set(kept)
        prev = kept


# --------------------------------------------------------------------------
# LoZA pattern (sink / recent / own chunk)
# --------------------------------------------------------------------------
def test_loza_select_worked_examples():
    # sink 2, recent 3, chunk 4, worked by hand from the three region rules
    pat = R.LozaPattern(sink=2, recent=3, chunk=4)
    expect = {0: [0], 3: [0, 1, 2, 3], 5: [0, 1, 3, 4, 5], 9: [0, 1, 7, 8, 9], 12: [0, 1, 10, 11, 12],
              15: [0, 1, 12, 13, 14, 15], 17: [0, 1, 15, 16, 17]}
    for p, keys in expect.items():
        assert R.loza_select(p, pat).tolist() == keys, p


@pytest.mark.parametrize("sink,recent,chunk", [(16, 1024, 4096), (2, 3, 4), (0, 1, 1), (5, 0, 7), (3, 9, 2),
                                               (0, 0, 5), (40, 8, 16)])
def test_loza_set_is_sink_plus_one_window(sink, recent, chunk):
    # every LoZA set is [0, min(sink, p+1)) followed by one run ending at p that
    # starts at the earlier of the recent window's and the chunk's first key
    pat = R.LozaPattern(sink=sink, recent=recent, chunk=chunk)
    for p in list(range(0, 70)) + [4095, 4096, 5119, 5120, 9000, 131071]:
        s_end = min(sink, p + 1)
        start = max(min(p - recent + 1, (p // chunk) * chunk), s_end)
        keys = list(range(s_end)) + list(range(start, p + 1))
        assert R.loza_select(p, pat).tolist() == keys, (sink, recent, chunk, p)


def test_loza_covering_window_is_dense_attention():
    rng = np.random.default_rng(41)
    qa = rng.standard_normal((32, 576))
    c = rng.standard_normal((300, 576))
    for p in (0, 7, 120, 299):
        for pat in (R.LozaPattern(sink=0, recent=p + 1, chunk=1), R.LozaPattern(sink=5, recent=1, chunk=512)):
            o, lse = R.loza_row(qa, c, p, pat)
            eo, el = R.dense_mla_row(qa, c, p)
            np.testing.assert_allclose(o, eo, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse, el, rtol=1e-12, atol=1e-12)


def test_loza_single_key_is_its_value_row():
    # sink 0, recent 1, chunk 1: only the query's own key, whose softmax weight is 1
    rng = np.random.default_rng(43)
    qa = rng.standard_normal((32, 576))
    c = rng.standard_normal((50, 576))
    pat = R.LozaPattern(sink=0, recent=1, chunk=1)
    for p in (0, 13, 49):
        o, lse = R.loza_row(qa, c, p, pat)
        np.testing.assert_array_equal(o, np.broadcast_to(c[p, :512], (32, 512)))
        np.testing.assert_allclose(lse, PAGES.softmax_scale * (qa @ c[p]), rtol=1e-12)
