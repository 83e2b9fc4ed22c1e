"""The C-ABI library loads, exports every symbol include/lsa.h declares, and its
host-side checks reject bad arguments before any CUDA call (CPU only)."""
import ctypes
import os
import re

import pytest

from sparse_attention_03_b200 import lsa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lsa.h")


@pytest.fixture(scope="module")
def lib():
    return lsa.load()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z0-9_]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("lsa_index_scores", "lsa_topk", "lsa_sparse_mla_decode", "lsa_sparse_mla_prefill",
                     "lsa_forward"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), f"{name} declared in lsa.h but not exported"
    assert set(lsa.EXPORTS) <= set(_declared())


def test_abi_version_and_defaults(lib):
    assert lib.lsa_abi_version() == 1
    c = lsa.Config()
    lib.lsa_config_default(ctypes.byref(c))
    assert (c.index_n_heads, c.index_head_dim, c.index_topk, c.index_init_tokens, c.index_local_tokens,
            c.cli_factor, c.n_heads, c.kv_lora_rank, c.qk_rope_head_dim) == (32, 128, 2048, 16, 1024, 2, 32, 512, 64)
    assert abs(c.softmax_scale - 192 ** -0.5) < 1e-7


def test_workspace_sizes(lib):
    cfg = lsa.LsaConfig()
    assert lsa.workspace_size(cfg, lsa.OP_TOPK, 64, 64, 1000) <= 256      # dense: nothing needed
    assert lsa.workspace_size(cfg, lsa.OP_TOPK, 64, 64, 32768) >= 64 * 40992
    big = lsa.workspace_size(cfg, lsa.OP_FORWARD_DECODE, 16, 16, 131072)
    assert big >= 16 * 131072 * 4        # the score rows
    pre = lsa.workspace_size(cfg, lsa.OP_FORWARD_PREFILL, 16384, 1, 16384)
    assert pre >= 16384 * 16384 * 4
    bad = lsa.LsaConfig(index_topk=10, index_init_tokens=5, index_local_tokens=5)
    assert lsa.workspace_size(bad, lsa.OP_TOPK, 4, 4, 100) == 0


def test_topk_workspace_grows_with_long_rows(lib):
    # few long rows (the multi-CTA select) keep up to a sixteenth of the row's
    # length of threshold-bin candidates (8 bytes each), at least the base 4096,
    # on top of the 8 KB histogram and control block of every row
    cfg = lsa.LsaConfig()
    base_row = 2056 * 4 + 4096 * 8                     # histogram + control, base candidates
    for rows, n in ((4, 983040), (16, 131072), (16, 40000), (3, 2 ** 23)):
        room = max(4096, min(n // 16, 2 ** 18))
        per = base_row + (room - 4096) * 8
        assert lsa.workspace_size(cfg, lsa.OP_TOPK, rows, rows, n) == rows * per + 256, (rows, n)
    # many rows or short rows take the one-CTA-per-row kernel: no candidate room
    assert lsa.workspace_size(cfg, lsa.OP_TOPK, 300, 300, 983040) == 300 * base_row + 256
    assert lsa.workspace_size(cfg, lsa.OP_TOPK, 4, 4, 16384) == 4 * base_row + 256


def _fake(n=1):
    return ctypes.c_void_p(0x10000 * n)  # aligned, never dereferenced by the host checks


def test_rejects_bad_config(lib):
    c = lsa.LsaConfig().c()
    c.index_n_heads = 16
    st = lib.lsa_index_scores(ctypes.byref(c), 4, 1, None, _fake(), _fake(), _fake(), _fake(), None, 100,
                              _fake(), 100, None, None)
    assert st == lsa.LSA_ERR_UNSUPPORTED
    assert b"32x128" in lib.lsa_last_error()
    st = lib.lsa_index_scores(None, 4, 1, None, _fake(), _fake(), _fake(), _fake(), None, 100, _fake(), 100, None,
                              None)
    assert st == lsa.LSA_ERR_INVALID


def test_rejects_bad_arguments(lib):
    c = lsa.LsaConfig().c()
    # ld < max_len
    assert lib.lsa_index_scores(ctypes.byref(c), 4, 1, None, _fake(), _fake(), _fake(), _fake(), None, 100,
                                _fake(), 50, None, None) == lsa.LSA_ERR_INVALID
    # misaligned q_idx
    assert lib.lsa_index_scores(ctypes.byref(c), 4, 1, None, _fake(), ctypes.c_void_p(0x10002), _fake(),
                                _fake(), None, 100, _fake(), 100, None, None) == lsa.LSA_ERR_INVALID
    # several sequences without offsets
    assert lib.lsa_index_scores(ctypes.byref(c), 4, 3, None, _fake(), _fake(), _fake(), _fake(), None, 100,
                                _fake(), 100, None, None) == lsa.LSA_ERR_INVALID
    # top-k without a workspace on few long rows (the multi-CTA path)
    assert lib.lsa_topk(ctypes.byref(c), 4, _fake(), 90000, _fake(), 90000, None, _fake(), _fake(), None, 0,
                        None) == lsa.LSA_ERR_WORKSPACE
    # a histogram buffer off the 16-byte grid (its per-row counters include a 64-bit one)
    assert lib.lsa_index_scores(ctypes.byref(c), 4, 1, None, _fake(), _fake(), _fake(), _fake(), None, 100,
                                _fake(), 100, ctypes.c_void_p(0x10004), None) == lsa.LSA_ERR_INVALID
    assert lib.lsa_topk(ctypes.byref(c), 4, _fake(), 90000, _fake(), 90000, ctypes.c_void_p(0x10004), _fake(),
                        _fake(), _fake(), 10 ** 7, None) == lsa.LSA_ERR_INVALID
    # decode MLA without offsets
    assert lib.lsa_sparse_mla_decode(ctypes.byref(c), 2, _fake(), _fake(), None, None, None, 10, _fake(),
                                     None, None, 0, None) == lsa.LSA_ERR_INVALID
    # forward: bad mode, prefill with several sequences
    arr = (ctypes.c_void_p * 2)(0x10000, 0x20000)
    assert lib.lsa_forward(ctypes.byref(c), 2, 1, 1, None, _fake(), 10, _fake(), _fake(), _fake(), _fake(),
                           arr, arr, arr, None, None, None, None, 0, None) == lsa.LSA_ERR_INVALID
    assert lib.lsa_forward(ctypes.byref(c), 1, 1, 2, None, _fake(), 10, _fake(), _fake(), _fake(), None,
                           arr, arr, arr, None, None, None, None, 0, None) == lsa.LSA_ERR_INVALID
    # sparse forward without workspace
    assert lib.lsa_forward(ctypes.byref(c), 0, 1, 1, None, _fake(), 5000, _fake(), _fake(), _fake(), _fake(),
                           arr, arr, arr, None, None, None, None, 0, None) == lsa.LSA_ERR_WORKSPACE


def test_empty_inputs_are_noops(lib):
    c = lsa.LsaConfig().c()
    assert lib.lsa_index_scores(ctypes.byref(c), 0, 1, None, None, None, None, None, None, 10, None, 10,
                                None, None) == lsa.LSA_OK
    assert lib.lsa_topk(ctypes.byref(c), 0, None, 10, None, 10, None, None, None, None, 0, None) == lsa.LSA_DENSE
    assert lib.lsa_sparse_mla_prefill(ctypes.byref(c), 0, None, None, None, 5, None, None, None, None, None,
                                      0, None) == lsa.LSA_OK


def test_index_project_validation(lib):
    c = lsa.LsaConfig().c()
    args = lambda q_lora, hidden, ws, theta=1.0e6: (ctypes.byref(c), 4, 1, None, _fake(), None, 100, _fake(), _fake(),
                                                    _fake(), _fake(), _fake(), _fake(), q_lora, hidden, theta,
                                                    _fake(), _fake(), _fake(), ws, 10 ** 9 if ws else 0, None)
    assert lib.lsa_index_project(*args(1536, 3000, _fake())) == lsa.LSA_ERR_INVALID     # hidden % 32
    assert b"multiples of 32" in lib.lsa_last_error()
    assert lib.lsa_index_project(*args(1536, 3072, None)) == lsa.LSA_ERR_WORKSPACE      # no workspace
    assert lib.lsa_index_project(*args(1536, 3072, _fake(), 0.5)) == lsa.LSA_ERR_INVALID
    assert lsa.workspace_size(lsa.LsaConfig(), lsa.OP_INDEX_PROJECT, 16, 16, 100) >= 16 * (4096 + 160) * 4


def test_hier_validation(lib):
    c = lsa.LsaConfig().c()
    f = _fake
    sel = lambda block, n_blocks, ws=None, wsb=0, k_blk=f(): (
        ctypes.byref(c), 4, 1, None, f(), f(), f(), f(), f(), k_blk, f(), 100000, block, n_blocks, f(), f(), ws,
        wsb, None)
    assert lib.lsa_hier_select(*sel(8, 500)) == lsa.LSA_ERR_UNSUPPORTED          # block below 16
    assert lib.lsa_hier_select(*sel(48 + 1, 100)) == lsa.LSA_ERR_UNSUPPORTED     # not a multiple of 16
    assert lib.lsa_hier_select(*sel(64, 31)) == lsa.LSA_ERR_UNSUPPORTED          # 31 x 64 < index_topk
    assert b"n_blocks * block" in lib.lsa_last_error()
    assert lib.lsa_hier_select(*sel(16, 2000)) == lsa.LSA_ERR_UNSUPPORTED        # coarse selection > 2048
    assert lib.lsa_hier_select(*sel(64, 32)) == lsa.LSA_ERR_WORKSPACE            # no workspace
    assert lib.lsa_hier_select(*sel(64, 32, f(), 10 ** 9, k_blk=None)) == lsa.LSA_ERR_INVALID
    n = lib.lsa_hier_workspace_size(ctypes.byref(c), 16, 131072, 64, 128)
    # coarse scores (2048 blocks) + compact rows ((1 + 17 + 128) x 64 slots) per row, fp32
    assert n >= 16 * (2048 + 146 * 64) * 4
    assert lib.lsa_hier_workspace_size(ctypes.byref(c), 16, 131072, 64, 10) == 0
    summ = lambda block, k_blk=f(): (ctypes.byref(c), 3, 2, f(), f(), f(), f(), f(), block, k_blk, None)
    assert lib.lsa_block_summaries(*summ(20)) == lsa.LSA_ERR_UNSUPPORTED
    assert lib.lsa_block_summaries(*summ(64, None)) == lsa.LSA_ERR_INVALID
    assert lsa.block_offsets([1, 64, 65, 0], 64) == [0, 1, 2, 4, 4]


def test_loza_validation(lib):
    c = lsa.LsaConfig().c()
    f = _fake()

    def call(pat, mode=0, k_off=f, n_seq=2, pos=f, seq=None):
        return lib.lsa_loza_mla(ctypes.byref(c), None if pat is None else ctypes.byref(lsa.LozaPattern(*pat)), mode,
                                3, n_seq, seq, pos, k_off, 100, f, f, f, None, None, 0, None)
    assert call(None) == lsa.LSA_ERR_INVALID
    assert call((16, 1024, 0)) == lsa.LSA_ERR_INVALID          # chunk < 1
    assert call((-1, 1024, 64)) == lsa.LSA_ERR_INVALID         # sink < 0
    assert call((16, -5, 64)) == lsa.LSA_ERR_INVALID           # recent < 0
    assert call((16, 1024, 64), k_off=None) == lsa.LSA_ERR_INVALID            # decode needs k_off
    assert call((16, 1024, 64), mode=1, n_seq=1) == lsa.LSA_ERR_INVALID       # prefill: k_off must be NULL
    assert call((16, 1024, 64), mode=1, k_off=None, n_seq=1, pos=None) == lsa.LSA_ERR_INVALID  # prefill needs pos
    assert call((16, 1024, 64), mode=2) == lsa.LSA_ERR_INVALID


def test_layer_and_mtp_attention_validation(lib):
    c = lsa.LsaConfig().c()
    f = _fake()
    arr = (ctypes.c_void_p * 4)(0x10000, 0x20000, 0x30000, 0x40000)
    bad = (ctypes.c_void_p * 2)(0x10000, 0x10002)              # the second pointer misaligned
    # both sub-blocks over one selection: NULL index list, NULL offsets, a misaligned sub-block pointer
    layer = lambda q, idx=f, k_off=f: lib.lsa_sparse_mla_decode_layer(ctypes.byref(c), 2, q, arr, k_off, idx, f,
                                                                       10, arr, None, None, 0, None)
    assert layer(arr, idx=None) == lsa.LSA_ERR_INVALID
    assert layer(arr, k_off=None) == lsa.LSA_ERR_INVALID
    assert layer(bad) == lsa.LSA_ERR_INVALID
    assert lib.lsa_sparse_mla_decode_layer(ctypes.byref(c), 0, None, None, None, None, None, 10, None, None, None,
                                           0, None) == lsa.LSA_OK
    # MTP: 1 <= n_draft <= 4, positions required
    mtp = lambda n, pos=f: lib.lsa_mtp_mla_decode(ctypes.byref(c), n, 2, pos, arr, f, f, f, f, 10, arr, None,
                                                  None, 0, None)
    assert mtp(0) == lsa.LSA_ERR_UNSUPPORTED
    assert mtp(5) == lsa.LSA_ERR_UNSUPPORTED
    assert b"n_draft" in lib.lsa_last_error()
    assert mtp(3, pos=None) == lsa.LSA_ERR_INVALID
    # split-K partials: fp32 [32 x 512] + (m, l) per head, for every (row, sub-block, split)
    cfg = lsa.LsaConfig()
    part = 32 * 512 * 4 + 32 * 8
    layer_ws = lsa.workspace_size(cfg, lsa.OP_MLA_DECODE_LAYER, 16, 16, 131072)
    assert layer_ws >= 16 * 2 * 2 * part                       # both sub-blocks, at least two splits each
    assert lsa.workspace_size(cfg, lsa.OP_MTP_DECODE, 16, 16, 131072) >= layer_ws   # sized for up to 4 steps


def test_wait_test_hook_is_one_shot_and_host_only(lib):
    # arming the hook touches no device; it applies to the next launch of the
    # thread only (consumed there), so arming twice before any launch is harmless
    lib.lsa_debug_arm_mla_wait_test(1000, 1)
    lib.lsa_debug_arm_mla_wait_test(0, -1)
