"""Seeded synthetic inputs for the LSA hot path (host side).

This module holds no part of the attention method's arithmetic. It only
draws numbers. Both the CPU oracle (through the tests) and the GPU harness use
it, and the CUDA library carries a second, independent implementation of the
same generator (``lsa_synth_*`` in the C-ABI) so that multi-gigabyte caches can
be drawn on the device and any sampled slice re-drawn here, bit for bit.

Definition of the generator
---------------------------
* Counter-based SplitMix64 (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014; Vigna's splitmix64.c).
  ``mix64(z)`` is the SplitMix64 output function. The stream of tensor
  ``tid`` under ``seed`` starts from the state
  ``key = mix64(seed ^ (tid * 0xD1B54A32D192ED03))`` and element ``i`` is the
  (i+1)-th SplitMix64 output from that state: ``mix64(key + (i+1) * GOLDEN)``.
* Approximate N(0, sigma^2): normal element ``i`` takes the stream's words
  ``2i`` and ``2i+1`` (outputs 2i+1 and 2i+2 from the key); their eight 16-bit
  fields are summed (Irwin-Hall, 8 terms), centred by subtracting 262140 and
  multiplied by one fp32 constant ``c = fp32(sigma / sqrt(2 (65536^2 - 1) / 3))``.
  The centred sum is an integer of magnitude at most 262140 < 2^18, exact in
  fp32, so the product is one correctly rounded fp32 multiply on any IEEE
  machine. Tails end at about 4.90 sigma (a true normal passes that once in
  about a million draws).
* bf16 values are the fp32 value rounded to nearest even.
* RMS-normalised rows (the index keys): the row is first rounded to bf16,
  then ``y = x / sqrt(sum(x^2)/d + 1e-6)``, evaluated in fp64 (the sum of the
  squares of bf16 values is exact in fp64, so its order does not matter),
  rounded to fp32 and then to bf16.
"""
from __future__ import annotations

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
TID_MUL = 0xD1B54A32D192ED03
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
IH_TERMS = 8
IH_VAR = 2.0 * (65536.0 * 65536.0 - 1.0) / 3.0  # variance of a sum of 8 uniform 16-bit ints
IH_CENTRE = 262140  # their mean, 8 * 65535 / 2

_U = np.uint64


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrap-around arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> _U(30))) * _U(M1)
        z = (z ^ (z >> _U(27))) * _U(M2)
    return z ^ (z >> _U(31))


def stream_key(seed: int, tid: int) -> int:
    s = (int(seed) ^ ((int(tid) * TID_MUL) & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
    return int(mix64(np.array([s], dtype=np.uint64))[0])


def hash_range(seed: int, tid: int, first: int, n: int) -> np.ndarray:
    """uint64 words for elements first .. first+n-1 of stream (seed, tid)."""
    key = _U(stream_key(seed, tid))
    i = np.arange(first + 1, first + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = key + i * _U(GOLDEN)
    return mix64(z)


def normal_scale(sigma: float) -> np.float32:
    """The single fp32 multiplier that maps the centred Irwin-Hall sum to N(0, sigma^2)."""
    return np.float32(float(sigma) / np.sqrt(IH_VAR))


def hash_at(seed: int, tid: int, index: np.ndarray) -> np.ndarray:
    """uint64 words for arbitrary element indices of stream (seed, tid)."""
    key = _U(stream_key(seed, tid))
    i = np.asarray(index, dtype=np.uint64) + _U(1)
    with np.errstate(over="ignore"):
        z = key + i * _U(GOLDEN)
    return mix64(z)


def _fields16(h: np.ndarray) -> np.ndarray:
    m = _U(0xFFFF)
    return (h & m) + ((h >> _U(16)) & m) + ((h >> _U(32)) & m) + ((h >> _U(48)) & m)


def _irwin_hall(h0: np.ndarray, h1: np.ndarray, sigma: float) -> np.ndarray:
    """Normal values from the two words of each element."""
    centred = (_fields16(h0) + _fields16(h1)).astype(np.int64) - IH_CENTRE
    return centred.astype(np.float32) * normal_scale(sigma)


def normal_f32_at(seed: int, tid: int, index: np.ndarray, sigma: float = 1.0) -> np.ndarray:
    i2 = 2 * np.asarray(index, dtype=np.int64)
    return _irwin_hall(hash_at(seed, tid, i2), hash_at(seed, tid, i2 + 1), sigma)


def normal_bf16_rows(seed: int, tid: int, rows: np.ndarray, d: int) -> np.ndarray:
    """bf16 bits [len(rows), d] of the given rows of a [*, d] normal tensor."""
    rows = np.asarray(rows, dtype=np.int64)
    index = rows[:, None] * d + np.arange(d, dtype=np.int64)[None, :]
    return f32_to_bf16_bits(normal_f32_at(seed, tid, index.ravel())).reshape(len(rows), d)


def normal_f32(seed: int, tid: int, first: int, n: int, sigma: float = 1.0) -> np.ndarray:
    h = hash_range(seed, tid, 2 * first, 2 * n)
    return _irwin_hall(h[0::2], h[1::2], sigma)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16, nearest even, returning the raw uint16 bits (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + _U(0x7FFF) + ((u >> _U(16)) & _U(1))
    return (u >> _U(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def normal_bf16(seed: int, tid: int, first: int, n: int, sigma: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0, sigma^2) draws."""
    return f32_to_bf16_bits(normal_f32(seed, tid, first, n, sigma))


def rms_rows_bf16(seed: int, tid: int, first_row: int, n_rows: int, d: int) -> np.ndarray:
    """bf16 bits [n_rows, d]: N(0,1) rows, rounded to bf16, then RMS-normalised."""
    bits = normal_bf16(seed, tid, first_row * d, n_rows * d).reshape(n_rows, d)
    x = bf16_bits_to_f64(bits)
    r = np.sqrt((x * x).sum(axis=1, keepdims=True) / d + 1e-6)
    y = (x / r).astype(np.float32)
    return f32_to_bf16_bits(y)


def uniform_int(seed: int, tid: int, first: int, n: int, lo: int, hi: int) -> np.ndarray:
    """Integers in [lo, hi] (inclusive): lo + (word mod (hi - lo + 1))."""
    h = hash_range(seed, tid, first, n)
    return (lo + (h % _U(hi - lo + 1)).astype(np.int64)).astype(np.int64)


# ---------------------------------------------------------------------------
# Tensor ids. One stream per tensor; per layer and attention sub-block.
# ---------------------------------------------------------------------------
Q_IDX, W, K_IDX, Q_ABS0, Q_ABS1, LAT0, LAT1, LENS = range(8)
# inputs of the indexer's own projections: q-LoRA vectors, hidden states, the
# weights wq_b / wk / weights_proj (N(0, 1/fan_in)) and the key-norm weight
C_Q, HIDDEN, WQ_B, WK, WPROJ, KNORM = range(8, 14)


def tid(layer: int, kind: int) -> int:
    return layer * 16 + kind


def q_abs_kind(sub: int) -> int:
    return (Q_ABS0, Q_ABS1)[sub]


def lat_kind(sub: int) -> int:
    return (LAT0, LAT1)[sub]


# The method's constants (index_n_heads, index_head_dim, n_heads, latent dims).
HI, DI, H, DLAT, DV = 32, 128, 32, 576, 512
W_SIGMA = 1.0 / np.sqrt(32.0)


def decode_lengths(seed: int, batch: int, lo: int, hi: int) -> np.ndarray:
    """Per-sequence cached lengths drawn uniformly in [lo, hi] (varlen decode batches)."""
    if lo == hi:
        return np.full(batch, lo, dtype=np.int64)
    return uniform_int(seed, tid(0, LENS), 0, batch, lo, hi)


def offsets(lengths: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lengths)
    return off


class Workload:
    """Host-side draw of one layer's inputs (small cases; big ones are drawn on the device).

    Decode: rows are sequences, ``pos[b] = L_b - 1``. Prefill: one sequence of
    ``n_keys`` keys and rows at positions ``q_start .. q_start + n_rows - 1``.
    Arrays are raw bf16 bits (uint16) or fp32.
    """

    def __init__(self, seed: int, layer: int, lengths, n_rows=None, q_start=None, cli=2):
        self.seed, self.layer, self.cli = seed, layer, cli
        self.lengths = np.asarray(lengths, dtype=np.int64)
        self.k_off = offsets(self.lengths)
        total = int(self.k_off[-1])
        if n_rows is None:  # decode
            self.mode = "decode"
            self.n_rows = len(self.lengths)
            self.seq_of_row = np.arange(self.n_rows, dtype=np.int32)
            self.pos = (self.lengths - 1).astype(np.int32)
        else:
            assert len(self.lengths) == 1
            self.mode = "prefill"
            self.n_rows = int(n_rows)
            self.seq_of_row = np.zeros(self.n_rows, dtype=np.int32)
            self.pos = (int(q_start) + np.arange(self.n_rows)).astype(np.int32)
        R = self.n_rows
        self.q_idx = normal_bf16(seed, tid(layer, Q_IDX), 0, R * HI * DI).reshape(R, HI, DI)
        self.w = normal_f32(seed, tid(layer, W), 0, R * HI, W_SIGMA).reshape(R, HI)
        self.k_idx = rms_rows_bf16(seed, tid(layer, K_IDX), 0, total, DI)
        self.q_abs = [normal_bf16(seed, tid(layer, q_abs_kind(z)), 0, R * H * DLAT).reshape(R, H, DLAT)
                      for z in range(cli)]
        self.latent = [normal_bf16(seed, tid(layer, lat_kind(z)), 0, total * DLAT).reshape(total, DLAT)
                       for z in range(cli)]
