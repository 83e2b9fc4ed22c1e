"""fp64 CPU oracle for the LongCat Sparse Attention (LSA) hot path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The product path (the
CUDA library and its Python binding) never calls it and shares no code with it.

Plain numpy float64, one query row at a time, in the order the pages state the
method. Sources (web pages; cited by title and section):

* [Lite-Sparse] "MLX-VLM 的 LongCat-Flash-Lite-Sparse 支持：LSA 稀疏注意力、
  n-gram 融合与预填充优化解析" (lmnt.cn). Sections used: "架构总览"
  (MLA dimensions), "LSA（LongCat 稀疏注意力）" (indexer, forcing, top-k,
  dense fallback, cross-layer reuse, gather vs mask), "预填充优化" (the
  ReLU-weighted head sum written as ``acc += max(g, 0) * w[h]``, and the
  unfused ``maximum(q k^T, 0)`` weighted-sum form), "测试与验证" (tiny
  config 8/2/4, absorbed == non-absorbed MLA).
* [LSA-2.0] "LongCat Sparse Attention技术深度解析：为什么它能提升100万上下文
  处理效率" (wmrh.cn). Sections used: "模型架构配置" (index_n_heads 32,
  index_head_dim 128, index_topk 2048, index_local_tokens 1024,
  index_init_tokens 16, cli_factor 2), "跨层索引" (one index pass serves
  consecutive layers), "多token预测模块集成" (the MTP draft steps share one
  index pass).

Readings taken where the pages are silent or garbled:
* The fallback comparison lost its operator in the scrape; it is read as
  "cached length <= index_topk", applied per query row.
* No extra scale in the index score; any scale lives in w.
* The local window is relative to each row: columns p-n_loc+1 .. p.
* Masking precedes forcing: columns after the query stay -inf.
* The query sees its own key (the cache is appended before indexing).
* Top-k is a set; ties are broken by the lower column index.
* Attention is MLA in absorbed form: logits use all 576 latent dims
  (512 c_kv + 64 rope), values are the first 512, scale 1/sqrt(128 + 64).

Parity pins for every function live in tests/test_oracle.py.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class LsaConfig:
    """Constants of the method ([LSA-2.0] 模型架构配置; [Lite-Sparse] 架构总览)."""

    index_topk: int = 2048
    index_init_tokens: int = 16
    index_local_tokens: int = 1024
    cli_factor: int = 2
    kv_lora_rank: int = 512          # value part of a latent row
    qk_rope_head_dim: int = 64
    qk_nope_head_dim: int = 128

    @property
    def softmax_scale(self) -> float:
        return 1.0 / np.sqrt(self.qk_nope_head_dim + self.qk_rope_head_dim)


PAGES = LsaConfig()
# The tiny configuration of the pages' language-model test ([Lite-Sparse] 测试与验证).
TINY = LsaConfig(index_topk=8, index_init_tokens=2, index_local_tokens=4, cli_factor=2)


def score_row(q: np.ndarray, w: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Lightning-indexer scores of one query against keys k.

    [Lite-Sparse] LSA section: q k per index head, then ReLU, then the sum over
    heads weighted by the per-head scalar; 预填充优化 gives the unfused form
    ``maximum(q k^T, 0)`` weighted sum, which is what this computes.

    q [Hi, d], w [Hi], k [n, d]  ->  s [n] with s[j] = sum_h w[h] * max(q[h].k[j], 0).
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    g = q @ k.T                       # [Hi, n]: one dot product per head and key
    return w @ np.maximum(g, 0.0)     # ReLU, then head-weighted sum


def mask_and_force(s_vis: np.ndarray, p: int, length: int, cfg: LsaConfig) -> np.ndarray:
    """Causal mask and streaming-aware forcing on one row of length ``length``.

    s_vis holds the scores of the visible columns 0..p. Columns after p become
    -inf (a query sees keys at positions <= its own). Of the visible columns,
    the first index_init_tokens (sink) and the last index_local_tokens (local
    window p-n_loc+1 .. p) become +inf ([Lite-Sparse] LSA section, streaming-
    aware indexing; [LSA-2.0] 模型架构配置).
    """
    out = np.full(length, -np.inf)
    out[: p + 1] = s_vis[: p + 1]
    j = np.arange(p + 1)
    forced = (j < cfg.index_init_tokens) | (j >= p + 1 - cfg.index_local_tokens)
    out[: p + 1][forced] = np.inf
    return out


def select_topk(s_row: np.ndarray, p: int, cfg: LsaConfig):
    """Top-k selection with the dense fallback ([Lite-Sparse] LSA section).

    If the query sees n = p+1 <= index_topk keys, the indexer returns nothing
    and attention is dense over all visible keys: returns (arange(n), True).
    Otherwise returns (the index_topk visible columns of highest score, ties to
    the lower index, False). The result is a set; its order carries no meaning.
    """
    n = p + 1
    if n <= cfg.index_topk:
        return np.arange(n, dtype=np.int64), True
    order = np.argsort(-s_row[:n], kind="stable")
    return np.sort(order[: cfg.index_topk]).astype(np.int64), False


def mla(q_abs: np.ndarray, c_sel: np.ndarray, cfg: LsaConfig):
    """Absorbed-latent MLA of one query over the selected latent rows.

    [Lite-Sparse] 架构总览 and LSA section: attention runs in the kv-LoRA latent
    space; keys are whole latent rows (c_kv 512 + rope 64), values are c_kv.
    q_abs [H, 576], c_sel [n, 576]  ->  o [H, 512], lse [H] (natural log).
    """
    q = np.asarray(q_abs, dtype=np.float64)
    c = np.asarray(c_sel, dtype=np.float64)
    x = cfg.softmax_scale * (q @ c.T)                 # [H, n] logits
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e / l) @ c[:, : cfg.kv_lora_rank]
    lse = (m + np.log(l))[:, 0]
    return o, lse


def lsa_row(q_idx, w, k_seq, p, q_abs_list, latent_list, cfg: LsaConfig = PAGES):
    """One query row through the whole path: index -> top-k -> cli_factor x MLA.

    k_seq [L, 128] and each latent [L, 576] hold the row's own sequence, with
    the current token already appended (the pages order the cache update before
    the gather). The index pass runs once and every sub-block reuses its
    selection ([Lite-Sparse] LSA section, cross-layer index reuse; [LSA-2.0]
    跨层索引). Returns (selected, dense, [(o, lse) per sub-block]).
    """
    L = k_seq.shape[0]
    n = p + 1
    if n <= cfg.index_topk:
        sel, dense = np.arange(n, dtype=np.int64), True     # the indexer is not run
    else:
        s = mask_and_force(score_row(q_idx, w, k_seq[:n]), p, L, cfg)
        sel, dense = select_topk(s, p, cfg)
    outs = [mla(qa, lat[sel], cfg) for qa, lat in zip(q_abs_list, latent_list)]
    return sel, dense, outs


def mtp_round(q_idx, w, k_seq, p, q_abs_steps, latent, cfg: LsaConfig = PAGES):
    """One round of multi-token-prediction drafting over one shared index pass.

    [LSA-2.0] 多token预测模块集成: the method extends to a three-step MTP module
    for speculative decoding, and all draft steps share a single index pass.
    Reading (the page says only that the pass is shared): the indexer, forcing
    and top-k (or the dense fallback) run once, for the first draft step's query
    at position p. Draft step i (i = 0, 1, ...) has its query at position p + i;
    by then the keys p+1 .. p+i (the earlier drafts' and its own) are in the
    cache, and a query sees its own key, so step i attends over the shared
    selection together with those keys. Nothing is dropped from the shared
    selection (it is reused as it stands).

    k_seq [L, 128] and latent [L, 576] hold the sequence's caches with keys
    0 .. p + len(q_abs_steps) - 1 present. Returns (selected, dense,
    [(o, lse) per step]).
    """
    n = p + 1
    if n <= cfg.index_topk:
        sel, dense = np.arange(n, dtype=np.int64), True      # the indexer is not run
    else:
        s = mask_and_force(score_row(q_idx, w, k_seq[:n]), p, k_seq.shape[0], cfg)
        sel, dense = select_topk(s, p, cfg)
    outs = []
    for i, qa in enumerate(q_abs_steps):
        keys = np.concatenate([sel, np.arange(p + 1, p + 1 + i, dtype=np.int64)])
        outs.append(mla(qa, latent[keys], cfg))
    return sel, dense, outs


def dense_mla_row(q_abs, latent, p, cfg: LsaConfig = PAGES):
    """Plain dense MLA over every visible key (attention_method MLA)."""
    return mla(q_abs, latent[: p + 1], cfg)


def explicit_mla(q_nope, q_rope, c_kv, k_rope, w_uk, w_uv, cfg: LsaConfig = PAGES):
    """Non-absorbed MLA, per head, for the absorbed == explicit self-check.

    k_h[i] = [W_UK[h] c[i] ; k_rope[i]], v_h[i] = W_UV[h] c[i]; softmax over i of
    scale * [q_nope[h]; q_rope[h]] . k_h[i]. ([Lite-Sparse] 测试与验证: the
    absorbed embed_q / unembed_out form must equal this.)
    q_nope [H,128], q_rope [H,64], c_kv [n,512], k_rope [n,64],
    w_uk [H,128,512], w_uv [H,128,512]  ->  out [H,128].
    """
    H = q_nope.shape[0]
    out = np.zeros((H, w_uv.shape[1]))
    for h in range(H):
        k = np.concatenate([c_kv @ w_uk[h].T, k_rope], axis=1)      # [n, 192]
        v = c_kv @ w_uv[h].T                                          # [n, 128]
        x = cfg.softmax_scale * (k @ np.concatenate([q_nope[h], q_rope[h]]))
        e = np.exp(x - x.max())
        out[h] = (e / e.sum()) @ v
    return out


def absorb_query(q_nope, q_rope, w_uk):
    """embed_q: fold W_UK into the query, q_abs[h] = [W_UK[h]^T q_nope[h] ; q_rope[h]]."""
    H = q_nope.shape[0]
    return np.stack([np.concatenate([w_uk[h].T @ q_nope[h], q_rope[h]]) for h in range(H)])


def unembed_out(o_lat, w_uv):
    """unembed_out: map each head's 512-d latent output back, out[h] = W_UV[h] o_lat[h]."""
    return np.stack([w_uv[h] @ o_lat[h] for h in range(o_lat.shape[0])])


# ---------------------------------------------------------------------------
# Upstream of the path: the indexer's own projections and the cache append.
# [Lite-Sparse] LSA section (the indexer's structure): wq_b maps the q-LoRA
# representation (q_lora_rank dims) to index_n_heads x index_head_dim; wk maps
# the hidden state to the index key, which is RMS-normalised; weights_proj
# gives one scalar per index head; the index query and key share MLA's RoPE
# configuration (qk_rope_head_dim, rope_theta).
# Readings (the pages leave these open): the RoPE part is the last
# qk_rope_head_dim dims of each 128-dim vector (MLA keeps its rope dims last),
# rotated in rotate-half form, pairs (i, i + rope/2) at angle
# pos * theta^(-2i/rope); no rope scaling; RMSNorm = x / sqrt(mean(x^2) + eps)
# times a per-dim weight, eps = 1e-6; no scale on the head weights.
# ---------------------------------------------------------------------------
Q_LORA, HIDDEN, ROPE_DIM, ROPE_THETA, NORM_EPS = 1536, 3072, 64, 1.0e6, 1e-6


def rope(x: np.ndarray, pos: float, theta: float = ROPE_THETA, rope_dim: int = ROPE_DIM) -> np.ndarray:
    """Rotary embedding of the last rope_dim dims of x[..., d] at position pos (fp64)."""
    x = np.array(x, dtype=np.float64)
    d = x.shape[-1]
    r0, half = d - rope_dim, rope_dim // 2
    ang = float(pos) * theta ** (-2.0 * np.arange(half) / rope_dim)
    c, s = np.cos(ang), np.sin(ang)
    a = x[..., r0:r0 + half].copy()
    b = x[..., r0 + half:].copy()
    x[..., r0:r0 + half] = a * c - b * s
    x[..., r0 + half:] = a * s + b * c
    return x


def rms_norm(x: np.ndarray, weight: np.ndarray, eps: float = NORM_EPS) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * weight


def index_project_row(c_q, h, wq_b, wk, wproj, k_norm_w, pos, theta=ROPE_THETA, eps=NORM_EPS):
    """One token's indexer inputs from its q-LoRA vector c_q [1536] and hidden
    state h [3072]: q_idx [32, 128] = RoPE(wq_b c_q), k [128] = RoPE(RMSNorm(wk h)),
    w [32] = weights_proj h. Weights are [out, in]."""
    q = (np.asarray(wq_b, np.float64) @ np.asarray(c_q, np.float64)).reshape(-1, 128)
    q = rope(q, pos, theta)
    k = rope(rms_norm(np.asarray(wk, np.float64) @ np.asarray(h, np.float64), k_norm_w, eps), pos, theta)
    w = np.asarray(wproj, np.float64) @ np.asarray(h, np.float64)
    return q, k, w


# ---------------------------------------------------------------------------
# Hierarchical indexing ([LSA-2.0] 分层索引): coarse-to-fine, two-stage scoring;
# approximate block-level scores first, then token-level selection inside the
# surviving blocks, so the indexer's candidate space shrinks.
# The page gives only that structure. Readings:
# * a block is `block` consecutive cached keys of one sequence (block b holds
#   positions b*block .. b*block + block - 1; the last one may be short);
# * a block's approximate score is the indexer's own score of the block's
#   summary key, the mean of its keys, rounded once to bf16 like every stored
#   key;
# * the coarse stage is the flat selection one level up: a row at position p
#   sees blocks 0 .. p // block; the ceil(n_init / block) sink blocks and the
#   ceil(n_loc / block) + 1 most recent blocks are forced in (together they
#   hold every forced token), and the n_blocks best of the others are kept,
#   ties to the lower block, with the same dense fallback (every block kept
#   when the row sees no more than that many);
# * the fine stage is the flat selection (mask, forcing, top-k, dense
#   fallback) over the tokens of the kept blocks only.
# ---------------------------------------------------------------------------
HIER_BLOCK, HIER_BLOCKS = 64, 128


def bf16_round(x) -> np.ndarray:
    """fp64 -> the nearest bf16 value (8 significant bits, ties to even), as fp64.
    Finite, normal-range inputs; computed on the fp64 bit pattern directly."""
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float64)).view(np.uint64)
    drop = np.uint64(52 - 7)                       # fp64 keeps 52 fraction bits, bf16 7
    half = np.uint64(1) << (drop - np.uint64(1))
    lsb = (b >> drop) & np.uint64(1)
    r = (b + half - np.uint64(1) + lsb) >> drop << drop
    return r.view(np.float64)


def block_summaries(k_seq: np.ndarray, block: int = HIER_BLOCK) -> np.ndarray:
    """Summary keys of every block of one sequence's cache k_seq [L, d]: the mean
    of the block's keys, rounded to bf16 -> [ceil(L / block), d]."""
    k = np.asarray(k_seq, dtype=np.float64)
    n = -(-k.shape[0] // block)
    return np.stack([bf16_round(k[b * block:(b + 1) * block].mean(axis=0)) for b in range(n)])


def hier_config(cfg: LsaConfig, block: int, n_blocks: int) -> LsaConfig:
    """The flat selection's constants one level up (blocks instead of tokens)."""
    n_init = -(-cfg.index_init_tokens // block)
    n_loc = -(-cfg.index_local_tokens // block) + 1
    return LsaConfig(index_topk=n_init + n_loc + n_blocks, index_init_tokens=n_init, index_local_tokens=n_loc,
                     cli_factor=cfg.cli_factor)


def hier_select(q, w, k_seq, k_blk, p, cfg: LsaConfig = PAGES, block: int = HIER_BLOCK,
                n_blocks: int = HIER_BLOCKS):
    """Hierarchical selection of one query row at position p over its sequence's
    keys k_seq [L, d] and block summaries k_blk [ceil(L / block), d].

    Returns (selected columns (sorted), dense flag, kept blocks (sorted)).
    """
    pb = p // block
    bcfg = hier_config(cfg, block, n_blocks)
    coarse = score_row(q, w, k_blk[: pb + 1])
    kept, _ = select_topk(mask_and_force(coarse, pb, pb + 1, bcfg), pb, bcfg)
    n = p + 1
    if n <= cfg.index_topk:
        return np.arange(n, dtype=np.int64), True, kept
    cand = np.concatenate([np.arange(b * block, min((b + 1) * block, n)) for b in kept])
    s = mask_and_force(score_row(q, w, k_seq[: p + 1]), p, p + 1, cfg)[cand]
    order = np.lexsort((cand, -s))                 # score descending, then lower column
    return np.sort(cand[order[: cfg.index_topk]]).astype(np.int64), False, kept


# --------------------------------------------------------------------------
# The LoZA sparse pattern ("LongCat-Flash-Thinking-ZigZag架构深度剖析",
# section "LoZA稀疏注意力机制" / "稀疏模式设计"): the attention matrix is split
# into a Sink region (the start of the sequence), a Recent region (the latest
# context) and a Chunked region (the middle, processed block by block). The
# page names the regions and no sizes. Reading: a query at position p attends
# to the keys j <= p with j < sink (Sink), p - j < recent (Recent), or
# j // chunk == p // chunk (its own chunk of the middle: Chunked); the set is
# static (no indexer) and attention over it is the same absorbed MLA.
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class LozaPattern:
    """Region sizes of the LoZA pattern (not given by the page; defaults are the
    LSA sink and local counts and a chunk of twice index_topk)."""

    sink: int = 16
    recent: int = 1024
    chunk: int = 4096


LOZA = LozaPattern()


def loza_select(p: int, pat: LozaPattern = LOZA) -> np.ndarray:
    """The keys a query at position p attends to, by the three region rules."""
    j = np.arange(p + 1)
    keep = (j < pat.sink) | (p - j < pat.recent) | (j // pat.chunk == p // pat.chunk)
    return j[keep]


def loza_row(q_abs: np.ndarray, latent: np.ndarray, p: int, pat: LozaPattern = LOZA, cfg: LsaConfig = PAGES):
    """Absorbed MLA of one query row over its LoZA set (latent rows 0..p of its sequence)."""
    return mla(q_abs, latent[loza_select(p, pat)], cfg)
