"""Python binding of liblsa.so (argument marshalling only).

Every function here takes torch tensors that live on a CUDA device, checks
their dtype, shape and contiguity, and passes raw pointers to the C entry point
of the same name (declared in include/lsa.h). All work runs in the library's
CUDA kernels on the current torch stream; there is no other implementation
behind these names. If the library is missing, load() raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsa.so")

LSA_OK, LSA_DENSE = 0, 1
LSA_ERR_INVALID, LSA_ERR_UNSUPPORTED, LSA_ERR_WORKSPACE, LSA_ERR_CUDA, LSA_ERR_DEVICE = -1, -2, -3, -4, -5
OP_TOPK, OP_MLA_DECODE, OP_MLA_PREFILL, OP_FORWARD_DECODE, OP_FORWARD_PREFILL = 1, 2, 3, 4, 5
OP_INDEX_PROJECT, OP_MLA_DECODE_LAYER, OP_MTP_DECODE = 6, 7, 8
TOPK_HIST_WORDS = 2056
DEVERR_POS, DEVERR_INDEX, DEVERR_COUNT, DEVERR_SEQ, DEVERR_TIMEOUT = 1, 2, 4, 8, 16

EXPORTS = (
    "lsa_config_default", "lsa_workspace_size", "lsa_index_scores", "lsa_topk",
    "lsa_sparse_mla_decode", "lsa_sparse_mla_prefill", "lsa_forward", "lsa_last_error",
    "lsa_device_error", "lsa_abi_version", "lsa_synth_normal_bf16", "lsa_synth_normal_f32",
    "lsa_synth_rms_rows_bf16", "lsa_launch_count", "lsa_index_project", "lsa_block_summaries",
    "lsa_hier_workspace_size", "lsa_hier_select", "lsa_sparse_mla_decode_topk", "lsa_loza_mla",
    "lsa_topk_static", "lsa_sparse_mla_decode_layer", "lsa_mtp_mla_decode", "lsa_debug_arm_mla_wait_test",
)
TOPK_STATIC_MAX_ROWS = 64
HIER_BLOCK, HIER_BLOCKS = 64, 128


class LsaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"status {status}: {msg}")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [
        ("index_n_heads", ctypes.c_int32),
        ("index_head_dim", ctypes.c_int32),
        ("index_topk", ctypes.c_int32),
        ("index_init_tokens", ctypes.c_int32),
        ("index_local_tokens", ctypes.c_int32),
        ("cli_factor", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("kv_lora_rank", ctypes.c_int32),
        ("qk_rope_head_dim", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
    ]


_lib = None
_P = ctypes.c_void_p
_I32, _I64, _U64, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t


def load():
    """Loads liblsa.so once. Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m sparse_attention_03_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.lsa_config_default.argtypes = [ctypes.POINTER(Config)]
    lib.lsa_config_default.restype = None
    lib.lsa_workspace_size.argtypes = [ctypes.POINTER(Config), _I32, _I32, _I32, _I64]
    lib.lsa_workspace_size.restype = _SZ
    lib.lsa_index_scores.argtypes = [ctypes.POINTER(Config), _I32, _I32, _P, _P, _P, _P, _P, _P, _I64, _P, _I64, _P,
                                     _P]
    lib.lsa_topk.argtypes = [ctypes.POINTER(Config), _I32, _P, _I64, _P, _I64, _P, _P, _P, _P, _SZ, _P]
    lib.lsa_topk_static.argtypes = [ctypes.POINTER(Config), _I32, _P, _I64, _P, _I64, _P, _P, _P]
    lib.lsa_sparse_mla_decode.argtypes = [ctypes.POINTER(Config), _I32, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _SZ, _P]
    lib.lsa_sparse_mla_decode_topk.argtypes = lib.lsa_sparse_mla_decode.argtypes
    _PP = ctypes.POINTER(_P)
    lib.lsa_sparse_mla_decode_layer.argtypes = [ctypes.POINTER(Config), _I32, _PP, _PP, _P, _P, _P, _I64, _PP, _PP,
                                                _P, _SZ, _P]
    lib.lsa_mtp_mla_decode.argtypes = [ctypes.POINTER(Config), _I32, _I32, _P, _PP, _P, _P, _P, _P, _I64, _PP, _PP,
                                       _P, _SZ, _P]
    lib.lsa_debug_arm_mla_wait_test.argtypes = [_I64, _I32]
    lib.lsa_debug_arm_mla_wait_test.restype = None
    lib.lsa_sparse_mla_prefill.argtypes = [ctypes.POINTER(Config), _I32, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _SZ, _P]
    lib.lsa_loza_mla.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(LozaPattern), _I32, _I32, _I32, _P, _P, _P,
                                 _I64, _P, _P, _P, _P, _P, _SZ, _P]
    lib.lsa_forward.argtypes = [ctypes.POINTER(Config), _I32, _I32, _I32, _P, _P, _I64, _P, _P, _P, _P,
                                ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_P),
                                _P, _P, _P, _SZ, _P]
    lib.lsa_index_project.argtypes = [ctypes.POINTER(Config), _I32, _I32, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _P,
                                      _I32, _I32, ctypes.c_float, _P, _P, _P, _P, _SZ, _P]
    lib.lsa_block_summaries.argtypes = [ctypes.POINTER(Config), _I32, _I32, _P, _P, _P, _P, _P, _I32, _P, _P]
    lib.lsa_hier_workspace_size.argtypes = [ctypes.POINTER(Config), _I32, _I64, _I32, _I32]
    lib.lsa_hier_workspace_size.restype = _SZ
    lib.lsa_hier_select.argtypes = [ctypes.POINTER(Config), _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _I32,
                                    _I32, _P, _P, _P, _SZ, _P]
    lib.lsa_last_error.argtypes = []
    lib.lsa_last_error.restype = ctypes.c_char_p
    lib.lsa_device_error.argtypes = [ctypes.POINTER(_I32)]
    lib.lsa_abi_version.argtypes = []
    lib.lsa_launch_count.argtypes = []
    lib.lsa_launch_count.restype = _I64
    lib.lsa_synth_normal_bf16.argtypes = [_P, _I64, _U64, _U64, _I64, ctypes.c_double, _P]
    lib.lsa_synth_normal_f32.argtypes = [_P, _I64, _U64, _U64, _I64, ctypes.c_double, _P]
    lib.lsa_synth_rms_rows_bf16.argtypes = [_P, _I64, _I32, _U64, _U64, _I64, _P]
    for name in ("lsa_index_scores", "lsa_topk", "lsa_topk_static", "lsa_sparse_mla_decode",
                 "lsa_sparse_mla_prefill", "lsa_sparse_mla_decode_layer", "lsa_mtp_mla_decode",
                 "lsa_forward", "lsa_index_project", "lsa_block_summaries", "lsa_hier_select", "lsa_device_error",
                 "lsa_sparse_mla_decode_topk", "lsa_loza_mla", "lsa_abi_version", "lsa_synth_normal_bf16",
                 "lsa_synth_normal_f32", "lsa_synth_rms_rows_bf16"):
        getattr(lib, name).restype = _I32
    _lib = lib
    return lib


@dataclass
class LsaConfig:
    index_topk: int = 2048
    index_init_tokens: int = 16
    index_local_tokens: int = 1024
    cli_factor: int = 2
    softmax_scale: float = 1.0 / (192.0 ** 0.5)

    def c(self) -> Config:
        """A fresh C struct of this configuration (safe to modify)."""
        cfg = Config()
        ctypes.pointer(cfg)[0] = self._c()
        return cfg

    def _c(self) -> Config:
        """The cached C struct passed to the library (never modified)."""
        key = (self.index_topk, self.index_init_tokens, self.index_local_tokens, self.cli_factor,
               self.softmax_scale)
        cfg = _CFG_CACHE.get(key)
        if cfg is None:
            cfg = Config()
            load().lsa_config_default(ctypes.byref(cfg))
            cfg.index_topk = self.index_topk
            cfg.index_init_tokens = self.index_init_tokens
            cfg.index_local_tokens = self.index_local_tokens
            cfg.cli_factor = self.cli_factor
            cfg.softmax_scale = self.softmax_scale
            _CFG_CACHE[key] = cfg
        return cfg


_CFG_CACHE: dict = {}


def _check(status: int, allow_dense: bool = False) -> int:
    if status < 0 or (status == LSA_DENSE and not allow_dense):
        raise LsaError(status, load().lsa_last_error().decode())
    return status


class Bound:
    """A C entry point with its arguments already marshalled: calling it only
    crosses the ABI (for tight host loops that must stay ahead of the GPU).
    The tensors it points at must outlive it; it launches on the stream that was
    current when it was bound."""

    __slots__ = ("fn", "args", "allow_dense", "keep")

    def __init__(self, fn, args, allow_dense, keep=None):
        self.fn, self.args, self.allow_dense, self.keep = fn, args, allow_dense, keep

    def __call__(self) -> int:
        st = self.fn(*self.args)
        if st < 0 or (st == LSA_DENSE and not self.allow_dense):
            raise LsaError(st, load().lsa_last_error().decode())
        return st


def _invoke(fn, args, allow_dense=False, bind=False, keep=None):
    if bind:
        return Bound(fn, args, allow_dense, keep)
    return _check(fn(*args), allow_dense)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dt(t, dtype, name):
    if t is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(cfg: LsaConfig, op: int, n_rows: int, n_seq: int, max_len: int) -> int:
    return int(load().lsa_workspace_size(ctypes.byref(cfg._c()), op, n_rows, n_seq, max_len))


def workspace(cfg: LsaConfig, op: int, n_rows: int, n_seq: int, max_len: int, device=None) -> torch.Tensor:
    n = workspace_size(cfg, op, n_rows, n_seq, max_len)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device or "cuda")


def topk_hist_buffer(n_rows, device=None) -> torch.Tensor:
    """A buffer for the optional top-k histogram lsa_index_scores can emit."""
    return torch.empty((n_rows, TOPK_HIST_WORDS), dtype=torch.int32, device=device or "cuda")


def index_scores(cfg, seq_of_row, pos, q_idx, w, k_idx, k_off, max_len, scores, n_seq=None, stream=None,
                 bind=False, topk_hist=None):
    _dt(q_idx, torch.bfloat16, "q_idx"); _dt(k_idx, torch.bfloat16, "k_idx"); _dt(w, torch.float32, "w")
    _dt(pos, torch.int32, "pos"); _dt(seq_of_row, torch.int32, "seq_of_row"); _dt(k_off, torch.int64, "k_off")
    _dt(scores, torch.float32, "scores")
    n_rows = pos.shape[0]
    if n_seq is None:
        n_seq = 1 if k_off is None else k_off.shape[0] - 1
    return _invoke(load().lsa_index_scores, (
        ctypes.byref(cfg._c()), n_rows, n_seq, _ptr(seq_of_row), _ptr(pos), _ptr(q_idx), _ptr(w),
        _ptr(k_idx), _ptr(k_off), int(max_len), _ptr(scores), scores.shape[1], _ptr(topk_hist), _stream(stream)),
        bind=bind)


def topk(cfg, pos, max_len, scores, idx, count, ws, stream=None, bind=False, topk_hist=None):
    _dt(scores, torch.float32, "scores"); _dt(pos, torch.int32, "pos")
    _dt(idx, torch.int32, "idx"); _dt(count, torch.int32, "count")
    return _invoke(load().lsa_topk, (
        ctypes.byref(cfg._c()), pos.shape[0], _ptr(pos), int(max_len), _ptr(scores), scores.shape[1],
        _ptr(topk_hist), _ptr(idx), _ptr(count), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
        allow_dense=True, bind=bind)


def topk_static(cfg, pos, max_len, scores, idx, count, stream=None, bind=False):
    """topk without a workspace: the library's built-in scratch (at most
    TOPK_STATIC_MAX_ROWS rows; calls that overlap on the GPU race on it)."""
    _dt(scores, torch.float32, "scores"); _dt(pos, torch.int32, "pos")
    _dt(idx, torch.int32, "idx"); _dt(count, torch.int32, "count")
    return _invoke(load().lsa_topk_static, (
        ctypes.byref(cfg._c()), pos.shape[0], _ptr(pos), int(max_len), _ptr(scores), scores.shape[1],
        _ptr(idx), _ptr(count), _stream(stream)), allow_dense=True, bind=bind)


def sparse_mla_decode(cfg, q_abs, latent, k_off, idx, count, max_len, out, lse, ws, stream=None, bind=False,
                      lists_from_topk=False):
    """Sparse absorbed MLA over each row's selected keys. lists_from_topk: idx /
    count were written by topk (or forward) for these rows and this config; the
    kernel then attends over the forced columns before the top-k has finished."""
    for t, n in ((q_abs, "q_abs"), (latent, "latent"), (out, "out")):
        _dt(t, torch.bfloat16, n)
    _dt(k_off, torch.int64, "k_off"); _dt(idx, torch.int32, "idx"); _dt(count, torch.int32, "count")
    _dt(lse, torch.float32, "lse")
    fn = load().lsa_sparse_mla_decode_topk if lists_from_topk else load().lsa_sparse_mla_decode
    return _invoke(fn, (
        ctypes.byref(cfg._c()), q_abs.shape[0], _ptr(q_abs), _ptr(latent), _ptr(k_off), _ptr(idx),
        _ptr(count), int(max_len), _ptr(out), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)), bind=bind)


def _bf16_list(ts, name):
    for t in ts:
        _dt(t, torch.bfloat16, name)
        _ptr(t)


def sparse_mla_decode_layer(cfg, q_abs, latent, k_off, idx, count, max_len, out, lse, ws, stream=None, bind=False):
    """The cfg.cli_factor sub-blocks sharing one top-k selection in one launch
    (q_abs, latent, out, lse: lists of cli_factor tensors; lse may be None)."""
    _bf16_list(list(q_abs) + list(latent) + list(out), "q_abs/latent/out")
    for t in (lse or []):
        _dt(t, torch.float32, "lse")
    _dt(k_off, torch.int64, "k_off"); _dt(idx, torch.int32, "idx"); _dt(count, torch.int32, "count")
    keep = (_ptr_array(q_abs), _ptr_array(latent), _ptr_array(out), _ptr_array(lse) if lse else None)
    return _invoke(load().lsa_sparse_mla_decode_layer, (
        ctypes.byref(cfg._c()), q_abs[0].shape[0], keep[0], keep[1], _ptr(k_off), _ptr(idx), _ptr(count),
        int(max_len), keep[2], keep[3], _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
        bind=bind, keep=keep)


def mtp_mla_decode(cfg, pos, q_abs, latent, k_off, idx, count, max_len, out, lse, ws, stream=None, bind=False):
    """The draft steps of one MTP round over one shared selection made at pos
    (q_abs, out, lse: lists of n_draft tensors; step i also sees keys pos+1..pos+i)."""
    _bf16_list(list(q_abs) + [latent] + list(out), "q_abs/latent/out")
    for t in (lse or []):
        _dt(t, torch.float32, "lse")
    _dt(pos, torch.int32, "pos"); _dt(k_off, torch.int64, "k_off"); _dt(idx, torch.int32, "idx")
    _dt(count, torch.int32, "count")
    keep = (_ptr_array(q_abs), _ptr_array(out), _ptr_array(lse) if lse else None)
    return _invoke(load().lsa_mtp_mla_decode, (
        ctypes.byref(cfg._c()), len(q_abs), pos.shape[0], _ptr(pos), keep[0], _ptr(latent), _ptr(k_off), _ptr(idx),
        _ptr(count), int(max_len), keep[1], keep[2], _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
        bind=bind, keep=keep)


def debug_arm_mla_wait_test(wait_ns: int, drop_tile: int):
    """Test hook: the next sparse-MLA launch of this thread stops issuing tiles at
    drop_tile and gives up its waits after wait_ns (see include/lsa.h)."""
    load().lsa_debug_arm_mla_wait_test(int(wait_ns), int(drop_tile))


def sparse_mla_prefill(cfg, pos, q_abs, latent, idx, count, out, lse, ws, stream=None, bind=False):
    for t, n in ((q_abs, "q_abs"), (latent, "latent"), (out, "out")):
        _dt(t, torch.bfloat16, n)
    _dt(pos, torch.int32, "pos"); _dt(idx, torch.int32, "idx"); _dt(count, torch.int32, "count")
    _dt(lse, torch.float32, "lse")
    return _invoke(load().lsa_sparse_mla_prefill, (
        ctypes.byref(cfg._c()), pos.shape[0], _ptr(pos), _ptr(q_abs), _ptr(latent), latent.shape[0],
        _ptr(idx), _ptr(count), _ptr(out), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)), bind=bind)


class LozaPattern(ctypes.Structure):
    """lsa_loza_pattern: sink keys, recent keys, chunk length."""
    _fields_ = [("sink", _I32), ("recent", _I32), ("chunk", _I32)]


def loza_mla(cfg, pattern, mode, seq_of_row, pos, k_off, max_len, q_abs, latent, out, lse, ws=None, stream=None,
             bind=False):
    """LoZA attention (sink, recent window, own chunk); pattern = (sink, recent, chunk)."""
    for t, n in ((q_abs, "q_abs"), (latent, "latent"), (out, "out")):
        _dt(t, torch.bfloat16, n)
    _dt(lse, torch.float32, "lse")
    pat = LozaPattern(*pattern)
    n_seq = 1 if k_off is None else k_off.shape[0] - 1
    return _invoke(load().lsa_loza_mla, (
        ctypes.byref(cfg._c()), ctypes.byref(pat), int(mode), q_abs.shape[0], n_seq, _ptr(seq_of_row), _ptr(pos),
        _ptr(k_off), int(max_len), _ptr(q_abs), _ptr(latent), _ptr(out), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel(), _stream(stream)), bind=bind, keep=(pat,))


def index_project(cfg, seq_of_row, pos, k_off, max_len, c_q, hidden, wq_b, wk, wproj, k_norm_w, q_idx, w, k_cache,
                  ws, rope_theta=1.0e6, stream=None, bind=False):
    """The indexer's q_idx [rows, 32, 128] and w [rows, 32] from c_q / hidden, and the
    rows' keys appended to k_cache (see lsa_index_project in include/lsa.h)."""
    for t, n in ((c_q, "c_q"), (hidden, "hidden"), (wq_b, "wq_b"), (wk, "wk"), (wproj, "wproj"),
                 (k_norm_w, "k_norm_w"), (q_idx, "q_idx"), (k_cache, "k_cache")):
        _dt(t, torch.bfloat16, n)
    _dt(w, torch.float32, "w"); _dt(pos, torch.int32, "pos")
    if seq_of_row is not None:
        _dt(seq_of_row, torch.int32, "seq_of_row")
    if k_off is not None:
        _dt(k_off, torch.int64, "k_off")
    n_seq = 1 if k_off is None else k_off.shape[0] - 1
    return _invoke(load().lsa_index_project, (
        ctypes.byref(cfg._c()), pos.shape[0], n_seq, _ptr(seq_of_row), _ptr(pos), _ptr(k_off), int(max_len),
        _ptr(c_q), _ptr(hidden), _ptr(wq_b), _ptr(wk), _ptr(wproj), _ptr(k_norm_w), c_q.shape[1], hidden.shape[1],
        float(rope_theta), _ptr(q_idx), _ptr(w), _ptr(k_cache), _ptr(ws), 0 if ws is None else ws.numel(),
        _stream(stream)), bind=bind)


def _ptr_array(ts):
    arr = (ctypes.c_void_p * len(ts))()
    for i, t in enumerate(ts):
        arr[i] = None if t is None else t.data_ptr()
    return arr


def forward(cfg, mode, seq_of_row, pos, max_len, q_idx, w, k_idx, k_off, q_abs, latent, out, lse,
            ws, idx_out=None, count_out=None, n_seq=None, stream=None, bind=False):
    """mode 0 decode / 1 prefill; q_abs, latent, out, lse: lists of cli_factor tensors."""
    for t in list(q_abs) + list(latent) + list(out):
        _dt(t, torch.bfloat16, "q_abs/latent/out")
        _ptr(t)
    for t in (lse or []):
        _dt(t, torch.float32, "lse")
        if t is not None:
            _ptr(t)
    if n_seq is None:
        n_seq = 1 if k_off is None else k_off.shape[0] - 1
    keep = (_ptr_array(q_abs), _ptr_array(latent), _ptr_array(out), _ptr_array(lse) if lse else None)
    return _invoke(load().lsa_forward, (
        ctypes.byref(cfg._c()), int(mode), pos.shape[0], n_seq, _ptr(seq_of_row), _ptr(pos), int(max_len),
        _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(k_off), keep[0], keep[1], keep[2], keep[3],
        _ptr(idx_out), _ptr(count_out), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)),
        bind=bind, keep=keep)


def launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(load().lsa_launch_count())


def device_error() -> int:
    """Synchronises, returns and clears the sticky device-side error flags."""
    flags = ctypes.c_int32(0)
    load().lsa_device_error(ctypes.byref(flags))
    return int(flags.value)


def synth_normal_bf16(dst, seed, tid, first=0, sigma=1.0, stream=None):
    _dt(dst, torch.bfloat16, "dst")
    return _check(load().lsa_synth_normal_bf16(_ptr(dst), dst.numel(), seed, tid, first, sigma, _stream(stream)))


def synth_normal_f32(dst, seed, tid, first=0, sigma=1.0, stream=None):
    _dt(dst, torch.float32, "dst")
    return _check(load().lsa_synth_normal_f32(_ptr(dst), dst.numel(), seed, tid, first, sigma, _stream(stream)))


def synth_rms_rows_bf16(dst, seed, tid, first_row=0, stream=None):
    _dt(dst, torch.bfloat16, "dst")
    n_rows, d = dst.shape
    return _check(load().lsa_synth_rms_rows_bf16(_ptr(dst), n_rows, d, seed, tid, first_row, _stream(stream)))


def block_offsets(lengths, block=HIER_BLOCK):
    """blk_off for packed caches of the given lengths: ceil(L / block) blocks each."""
    n = [(int(L) + block - 1) // block for L in lengths]
    off = [0]
    for x in n:
        off.append(off[-1] + x)
    return off


def block_summaries(cfg, item_seq, item_blk, k_idx, k_off, blk_off, k_blk, block=HIER_BLOCK, stream=None,
                    bind=False):
    """Summary keys (bf16 mean of the block's keys) of blocks item_blk[i] of
    sequences item_seq[i] into k_blk (hierarchical indexing)."""
    _dt(k_idx, torch.bfloat16, "k_idx"); _dt(k_blk, torch.bfloat16, "k_blk")
    _dt(item_seq, torch.int32, "item_seq"); _dt(item_blk, torch.int32, "item_blk")
    _dt(k_off, torch.int64, "k_off"); _dt(blk_off, torch.int64, "blk_off")
    return _invoke(load().lsa_block_summaries, (
        ctypes.byref(cfg._c()), item_seq.numel(), k_off.numel() - 1, _ptr(item_seq), _ptr(item_blk), _ptr(k_idx),
        _ptr(k_off), _ptr(blk_off), block, _ptr(k_blk), _stream(stream)), bind=bind)


def hier_workspace(cfg, n_rows, max_len, block=HIER_BLOCK, n_blocks=HIER_BLOCKS, device=None) -> torch.Tensor:
    n = int(load().lsa_hier_workspace_size(ctypes.byref(cfg._c()), n_rows, max_len, block, n_blocks))
    if n == 0:
        raise LsaError(LSA_ERR_UNSUPPORTED, load().lsa_last_error().decode())
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def hier_select(cfg, seq_of_row, pos, q_idx, w, k_idx, k_off, k_blk, blk_off, max_len, idx, count, ws,
                block=HIER_BLOCK, n_blocks=HIER_BLOCKS, stream=None, bind=False):
    """Two-stage (block, then token) selection of every row into idx / count,
    shaped like topk's output."""
    _dt(q_idx, torch.bfloat16, "q_idx"); _dt(k_idx, torch.bfloat16, "k_idx"); _dt(k_blk, torch.bfloat16, "k_blk")
    _dt(w, torch.float32, "w"); _dt(pos, torch.int32, "pos"); _dt(idx, torch.int32, "idx")
    _dt(count, torch.int32, "count"); _dt(k_off, torch.int64, "k_off"); _dt(blk_off, torch.int64, "blk_off")
    _dt(seq_of_row, torch.int32, "seq_of_row")
    return _invoke(load().lsa_hier_select, (
        ctypes.byref(cfg._c()), pos.numel(), k_off.numel() - 1, _ptr(seq_of_row), _ptr(pos), _ptr(q_idx), _ptr(w),
        _ptr(k_idx), _ptr(k_off), _ptr(k_blk), _ptr(blk_off), int(max_len), block, n_blocks, _ptr(idx),
        _ptr(count), _ptr(ws), ws.numel(), _stream(stream)), allow_dense=True, bind=bind)
