"""lsa_topk_static, the top-k entry point for callers that cannot allocate
device memory (graph capture, allocation-free serving loops, plugins given only
their buffers), must select exactly what lsa_topk selects with a caller
workspace, on consecutive calls that share its built-in scratch.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

MAX_ROWS = 64


def _scores(seed):
    rng = np.random.default_rng(seed)
    pos = np.concatenate([[0, 700, 2047, 2048, 2049, 5000], rng.integers(2100, 150000, 34)]).astype(np.int32)
    max_len = int(pos.max()) + 1
    s = np.full((len(pos), max_len), -np.inf, dtype=np.float32)
    for r, p in enumerate(pos):
        v = rng.standard_normal(p + 1).astype(np.float32) * 8
        if r % 5 == 0:
            v = np.round(v)          # ties
        s[r, : p + 1] = v
    return pos, max_len, s


def _call_static(lib, cfg, pos, max_len, scores, idx, cnt):
    return lib.lsa_topk_static(ctypes.byref(cfg), int(pos.shape[0]), ctypes.c_void_p(pos.data_ptr()),
                               int(max_len), ctypes.c_void_p(scores.data_ptr()), int(scores.shape[1]),
                               ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_topk_static_matches_topk_on_two_calls():
    from sparse_attention_03_b200 import lsa
    lib = lsa.load()
    lib.lsa_topk_static.argtypes = [ctypes.POINTER(lsa.Config), ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64,
                                    ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p]
    lib.lsa_topk_static.restype = ctypes.c_int32
    pycfg = lsa.LsaConfig()
    cfg = pycfg.c()
    for call, seed in enumerate((1, 2)):
        pos_h, max_len, s_h = _scores(seed)
        n = len(pos_h)
        pos = torch.from_numpy(pos_h).cuda()
        scores = torch.from_numpy(s_h).cuda()
        ref_idx = torch.empty((n, 2048), dtype=torch.int32, device="cuda")
        ref_cnt = torch.empty((n,), dtype=torch.int32, device="cuda")
        ws = lsa.workspace(pycfg, lsa.OP_TOPK, n, n, max_len)
        lsa.topk(pycfg, pos, max_len, scores, ref_idx, ref_cnt, ws)
        idx = torch.full((n, 2048), -9, dtype=torch.int32, device="cuda")
        cnt = torch.full((n,), -9, dtype=torch.int32, device="cuda")
        assert _call_static(lib, cfg, pos, max_len, scores, idx, cnt) == lsa.LSA_OK, lib.lsa_last_error()
        torch.cuda.synchronize()
        a, b = ref_idx.cpu().numpy(), idx.cpu().numpy()
        np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt.cpu().numpy())
        for r in range(n):
            np.testing.assert_array_equal(np.sort(b[r]), np.sort(a[r]), err_msg=f"call {call} row {r}")
    assert lsa.device_error() == 0


def test_topk_static_rejects_too_many_rows():
    from sparse_attention_03_b200 import lsa
    lib = lsa.load()
    lib.lsa_topk_static.restype = ctypes.c_int32
    cfg = lsa.LsaConfig().c()
    st = lib.lsa_topk_static(ctypes.byref(cfg), MAX_ROWS + 1, ctypes.c_void_p(16), 5000, ctypes.c_void_p(16),
                             5000, ctypes.c_void_p(16), ctypes.c_void_p(16), None)
    assert st == lsa.LSA_ERR_INVALID
    assert b"exceed" in lib.lsa_last_error()
