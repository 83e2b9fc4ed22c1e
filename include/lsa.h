/*
 * lsa.h - C-ABI of liblsa.so, the B200 (sm_100a) hot path of LongCat Sparse
 * Attention (LSA): lightning indexer -> top-k with forced sink/local columns
 * and a dense fallback -> absorbed-latent MLA over the selected keys, with one
 * index pass shared by a layer's attention sub-blocks.
 *
 * Sources (web pages, cited by title and section):
 *   [Lite-Sparse] "MLX-VLM 的 LongCat-Flash-Lite-Sparse 支持：LSA 稀疏注意力、
 *     n-gram 融合与预填充优化解析", sections "架构总览",
 *     "LSA（LongCat 稀疏注意力）", "预填充优化", "测试与验证".
 *   [LSA-2.0] "LongCat Sparse Attention技术深度解析：为什么它能提升100万上下文
 *     处理效率", sections "流式感知索引", "跨层索引", "模型架构配置".
 *   "LongCat-Flash-Thinking-ZigZag架构深度剖析", section "LoZA稀疏注意力机制"
 *     (lsa_loza_mla only).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every array argument is DEVICE memory owned by the caller, unless stated
 *   otherwise. The library never allocates, frees or synchronises (except the
 *   two debugging calls marked "synchronising"). All work is enqueued on
 *   `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream).
 * - lsa_bf16 is the raw 16-bit pattern of a bfloat16 value.
 * - Row-major layouts. Index vectors: 128 bf16 = 256 B per key. Latent rows:
 *   576 bf16 = 1152 B (512 c_kv then 64 rope). Bases of bf16 arrays must be
 *   16-byte aligned.
 * - Sequences: the keys of sequence b are rows [k_off[b], k_off[b+1]) of the
 *   packed caches (k_off: int64 [n_seq+1], device). Query row r belongs to
 *   sequence seq_of_row[r] and sits at absolute position pos[r] inside it; it
 *   sees keys 0..pos[r] (its own key included: the caller appends the current
 *   token's cache rows before calling, as the pages order the cache update
 *   before the gather).
 * - Errors: host-detectable errors return at once and enqueue nothing
 *   (LSA_ERR_INVALID, LSA_ERR_UNSUPPORTED, LSA_ERR_WORKSPACE); a failed launch
 *   returns LSA_ERR_CUDA. Device-detected errors (a position past its
 *   sequence, an index out of range) never fault: the kernel clamps or skips
 *   the bad item and sets a sticky flag read by lsa_device_error().
 *   lsa_last_error() gives a message for the last failing call on the thread.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LSA_API __attribute__((visibility("default")))
#else
#define LSA_API
#endif

typedef uint16_t lsa_bf16;

typedef enum lsa_status {
  LSA_OK = 0,
  LSA_DENSE = 1,             /* lsa_topk: every row is dense (no selection needed) */
  LSA_ERR_INVALID = -1,      /* null pointer, bad size, misalignment */
  LSA_ERR_UNSUPPORTED = -2,  /* configuration the kernels do not implement */
  LSA_ERR_WORKSPACE = -3,    /* ws_bytes below the minimum */
  LSA_ERR_CUDA = -4,         /* a CUDA call or launch failed */
  LSA_ERR_DEVICE = -5        /* lsa_device_error() found a device-side flag */
} lsa_status;

/* Device-side error flags (lsa_device_error). */
#define LSA_DEVERR_POS 1     /* pos[r] < 0 or beyond its sequence or max_len */
#define LSA_DEVERR_INDEX 2   /* a selected index outside the row's visible keys */
#define LSA_DEVERR_COUNT 4   /* count[r] outside [0, index_topk] */
#define LSA_DEVERR_SEQ 8     /* seq_of_row[r] outside [0, n_seq) */
#define LSA_DEVERR_TIMEOUT 16 /* a bounded wait inside a kernel gave up (the CTA stopped early) */

/*
 * Method constants, under the pages' config key names ([LSA-2.0] 模型架构配置;
 * [Lite-Sparse] 架构总览). Supported: index_n_heads 32, index_head_dim 128,
 * n_heads 32, kv_lora_rank 512, qk_rope_head_dim 64, cli_factor 1 or 2,
 * 0 <= index_init_tokens, 0 <= index_local_tokens,
 * index_init_tokens + index_local_tokens < index_topk <= 2048.
 */
typedef struct lsa_config {
  int32_t index_n_heads;      /* 32 */
  int32_t index_head_dim;     /* 128 */
  int32_t index_topk;         /* 2048 */
  int32_t index_init_tokens;  /* 16: sink columns forced into the selection */
  int32_t index_local_tokens; /* 1024: local-window columns forced in */
  int32_t cli_factor;         /* 2: attention sub-blocks sharing one index pass */
  int32_t n_heads;            /* 32 MLA heads */
  int32_t kv_lora_rank;       /* 512: value part of a latent row */
  int32_t qk_rope_head_dim;   /* 64: rope part of a latent row */
  float softmax_scale;        /* 1/sqrt(qk_nope 128 + qk_rope 64) */
} lsa_config;

/* Fills the pages' constants (the values in the comments above). */
LSA_API void lsa_config_default(lsa_config* cfg);

/* Operation codes for lsa_workspace_size. */
#define LSA_OP_TOPK 1
#define LSA_OP_MLA_DECODE 2
#define LSA_OP_MLA_PREFILL 3
#define LSA_OP_FORWARD_DECODE 4
#define LSA_OP_FORWARD_PREFILL 5
#define LSA_OP_INDEX_PROJECT 6
#define LSA_OP_MLA_DECODE_LAYER 7 /* lsa_sparse_mla_decode_layer (cfg->cli_factor sub-blocks) */
#define LSA_OP_MTP_DECODE 8       /* lsa_mtp_mla_decode (any n_draft) */

/*
 * Bytes of workspace the operation uses at full speed for these sizes (host
 * only, no CUDA call). Smaller workspaces are accepted down to a minimum
 * (one row block for top-k and forward; zero for the MLA calls, which then
 * run without split-K); below it the call returns LSA_ERR_WORKSPACE.
 * Returns 0 on invalid arguments.
 */
LSA_API size_t lsa_workspace_size(const lsa_config* cfg, int32_t op, int32_t n_rows, int32_t n_seq,
                          int64_t max_len);

/*
 * Lightning-indexer scores, mask and forcing ([Lite-Sparse] LSA section: q k
 * per index head, ReLU, head-weighted sum; streaming-aware forcing; 预填充优化:
 * the fused ReLU-weighted epilogue that never materialises the per-head
 * tensor).
 *
 *   scores[r, j] = sum_h w[r,h] * max(q_idx[r,h,:] . k_idx[k_off[b] + j, :], 0)
 *                  for j <= pos[r], b = seq_of_row[r];
 *                = +inf  if j <= pos[r] and (j < index_init_tokens or
 *                        j > pos[r] - index_local_tokens)   (forced columns).
 * Entries at j > pos[r] are not written: the causal mask is applied by never
 * reading them (lsa_topk reads columns 0..pos[r] only).
 *
 * q_idx   bf16 [n_rows, 32, 128]     w  fp32 [n_rows, 32]
 * k_idx   bf16 [sum L_b, 128]        k_off int64 [n_seq+1], or NULL: one
 *         sequence of max_len keys at row 0 (then n_seq must be 1)
 * seq_of_row int32 [n_rows] or NULL (every row in sequence 0)
 * pos     int32 [n_rows]             scores fp32 [n_rows, ld], ld >= max_len
 * max_len host bound: every pos[r] < max_len.
 * topk_hist: optional uint32 [n_rows, LSA_TOPK_HIST_WORDS] (device, 16-byte
 *   aligned). When not NULL it receives the first radix pass of the selection (a histogram of the
 *   top 11 bits of the order-preserving key of every middle-column score of
 *   rows with more than index_topk visible keys), built from the scores while
 *   they are still in registers; pass it to lsa_topk with the same scores.
 * Products bf16 x bf16 exact in fp32, fp32 accumulation.
 */
#define LSA_TOPK_HIST_WORDS 2056 /* uint32 words per row of a top-k histogram buffer */
LSA_API lsa_status lsa_index_scores(const lsa_config* cfg, int32_t n_rows, int32_t n_seq,
                            const int32_t* seq_of_row, const int32_t* pos, const lsa_bf16* q_idx,
                            const float* w, const lsa_bf16* k_idx, const int64_t* k_off,
                            int64_t max_len, float* scores, int64_t ld, uint32_t* topk_hist,
                            void* stream);

/*
 * Top-k selection with the dense fallback ([Lite-Sparse] LSA section: the
 * index_topk columns of highest score; the forced columns always enter; when
 * the cached length is <= index_topk the indexer yields nothing and attention
 * is dense).
 *
 * Row r with n = pos[r]+1 visible columns:
 *   n <= index_topk: idx[r, :n] = 0..n-1, idx[r, n:] = -1, count[r] = n;
 *   otherwise: count[r] = index_topk and idx[r, :] holds, unordered, the
 *   index_init_tokens sink columns, the index_local_tokens local columns and
 *   the remaining columns of highest score (ties to the lower index).
 * scores fp32 [n_rows, ld] as written by lsa_index_scores (only columns
 * 0..pos[r] are read). idx int32 [n_rows, index_topk], count int32 [n_rows].
 * max_len (host): every pos[r] < max_len. Returns LSA_DENSE when
 * max_len <= index_topk (every row dense; idx/count still written).
 * topk_hist: NULL, or the histogram lsa_index_scores wrote for these scores
 *   (saves one pass over the scores; 16-byte aligned, else LSA_ERR_INVALID).
 *   Rows longer than 16384 columns (fewer than 256 rows) also keep their
 *   counters in its 8 words after each row's bins (one of them a 64-bit
 *   counter): they must be zero on entry, as lsa_index_scores leaves them, and
 *   are zero again on return.
 * Workspace: lsa_workspace_size(LSA_OP_TOPK, ...). Only fewer than 256 rows
 * longer than 16384 columns use it (then processed in blocks that fit,
 * minimum one row of 40992 B); otherwise ws may be NULL.
 */
LSA_API lsa_status lsa_topk(const lsa_config* cfg, int32_t n_rows, const int32_t* pos, int64_t max_len,
                    const float* scores, int64_t ld, uint32_t* topk_hist, int32_t* idx,
                    int32_t* count, void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_topk_static: the same selection as lsa_topk, for callers that cannot
 * allocate device memory. The pages have no counterpart of this entry point.
 *
 * Who needs it: code being recorded into a CUDA graph (an allocation is not a
 * stream operation, so a capture cannot contain one), serving loops that must
 * not pay the device-wide synchronisation cudaMalloc/cudaFree may cause, and
 * plugins whose host framework hands them only their input and output buffers.
 * The caller passes the buffers of lsa_topk except the workspace and the
 * optional topk_hist (this entry point always builds its own histogram).
 *
 * Scratch: a file-scope device array of LSA_TOPK_STATIC_MAX_ROWS x 40992 bytes
 * (2.5 MiB) inside the library; every GPU that loads the library keeps it
 * until the process exits. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current: make that
 * first call before any stream capture begins. The call allocates nothing.
 * All calls share the one array and each call clears what must start at
 * zero; calls whose kernels may overlap on the GPU (other streams, other host
 * threads) race on it and must be serialised by the caller.
 * n_rows > LSA_TOPK_STATIC_MAX_ROWS returns LSA_ERR_INVALID (split the rows or
 * use lsa_topk). The configuration is checked as lsa_topk checks it; statuses
 * otherwise as lsa_topk.
 */
#define LSA_TOPK_STATIC_MAX_ROWS 64
LSA_API lsa_status lsa_topk_static(const lsa_config* cfg, int32_t n_rows, const int32_t* pos,
                                   int64_t max_len, const float* scores, int64_t ld, int32_t* idx,
                                   int32_t* count, void* stream);

/*
 * The indexer's own inputs from the model's activations, and the key-cache
 * append ([Lite-Sparse] LSA section, the indexer's structure: wq_b maps the
 * q-LoRA representation to index_n_heads x index_head_dim, wk maps the hidden
 * state to the index key, which is RMS-normalised (index_k_norm_type rms),
 * weights_proj gives one scalar per index head, and the index query and key
 * share MLA's RoPE configuration (qk_rope_head_dim, rope_theta)). This is
 * upstream of lsa_index_scores; it feeds its q_idx, w and k_idx.
 *
 * For each row r (sequence seq_of_row[r], position pos[r]):
 *   q_idx[r,h,:] = RoPE(wq_b c_q[r])[h*128 .. h*128+127]          (bf16 out)
 *   w[r,:]       = weights_proj hidden[r]                           (fp32 out)
 *   k_cache[k_off[seq] + pos[r], :] = RoPE(RMSNorm(wk hidden[r]))   (bf16 out)
 * RoPE rotates the last qk_rope_head_dim (64) dims of each 128-dim vector in
 * rotate-half form: pairs (i, i+32) by pos * rope_theta^(-2i/64). RMSNorm:
 * x / sqrt(mean(x^2) + 1e-6) * k_norm_w. These readings fill what the pages
 * leave open (which dims carry RoPE, its form, the epsilon); no rope scaling.
 * c_q bf16 [n_rows, q_lora_rank]; hidden bf16 [n_rows, hidden_size]; wq_b bf16
 * [32*128, q_lora_rank]; wk bf16 [128, hidden_size]; wproj bf16 [32,
 * hidden_size]; k_norm_w bf16 [128]; q_idx bf16 [n_rows, 32, 128]; w fp32
 * [n_rows, 32]; k_cache bf16 packed [sum L, 128] (only the rows' own slots are
 * written). q_lora_rank and hidden_size must be positive multiples of 32; every
 * pointer 16-byte aligned. seq_of_row NULL: row r is sequence r when k_off is
 * given, else every row is sequence 0 with k_cache rows = positions. max_len
 * (host) bounds every position. A row whose sequence or position is out of
 * range writes no cache row and raises a device error flag.
 * Workspace (fp32 products): lsa_workspace_size(LSA_OP_INDEX_PROJECT).
 */
LSA_API lsa_status lsa_index_project(const lsa_config* cfg, int32_t n_rows, int32_t n_seq,
                                     const int32_t* seq_of_row, const int32_t* pos, const int64_t* k_off,
                                     int64_t max_len, const lsa_bf16* c_q, const lsa_bf16* hidden,
                                     const lsa_bf16* wq_b, const lsa_bf16* wk, const lsa_bf16* wproj,
                                     const lsa_bf16* k_norm_w, int32_t q_lora_rank, int32_t hidden_size,
                                     float rope_theta, lsa_bf16* q_idx, float* w, lsa_bf16* k_cache, void* ws,
                                     size_t ws_bytes, void* stream);

/*
 * Hierarchical indexing ([LSA-2.0] "分层索引": coarse-to-fine two-stage
 * scoring, approximate block-level scores first, then token selection inside
 * the surviving blocks, so the indexer handles a smaller candidate space).
 * The page gives only that structure; the readings taken are: a block is
 * `block` consecutive cached keys of one sequence; its summary key is the mean
 * of its keys rounded once to bf16; the coarse stage is the flat selection one
 * level up (the ceil(init/block) sink blocks and the ceil(local/block) + 1 most
 * recent blocks forced in, the n_blocks best other blocks kept, ties to the
 * lower block, every block kept when the row sees no more than that many); the
 * fine stage is the flat selection (mask, forcing, top-k, dense fallback) over
 * the tokens of the kept blocks.
 *
 * lsa_block_summaries: for each item i, the summary of block item_blk[i] of
 * sequence item_seq[i] (the mean of its keys at positions < the sequence's
 * length, in fp64, rounded to nearest-even bf16). Call it for every block at
 * build time and, after each append, for the block holding the new key.
 *   k_idx: packed [sum L, 128] bf16 with k_off int64 [n_seq+1] (as lsa_index_scores).
 *   blk_off: int64 [n_seq+1], blk_off[s+1] - blk_off[s] >= ceil(L_s / block).
 *   k_blk: packed [blk_off[n_seq], 128] bf16 (16-byte aligned), caller-owned.
 *   block: 16 .. 1024, a multiple of 16.
 * An item naming a sequence or block out of range is skipped and sets
 * LSA_DEVERR_SEQ / LSA_DEVERR_POS.
 */
LSA_API lsa_status lsa_block_summaries(const lsa_config* cfg, int32_t n_items, int32_t n_seq,
                                       const int32_t* item_seq, const int32_t* item_blk, const lsa_bf16* k_idx,
                                       const int64_t* k_off, const int64_t* blk_off, int32_t block,
                                       lsa_bf16* k_blk, void* stream);

/*
 * lsa_hier_select: the two-stage selection of every row, output as lsa_topk's
 * (idx int32 [n_rows, index_topk] unordered, count int32 [n_rows]; rows with
 * pos + 1 <= index_topk are dense: 0..pos).
 *   Rows, queries and keys as lsa_index_scores (seq_of_row NULL: sequence 0);
 *   k_blk / blk_off as written by lsa_block_summaries for the same caches.
 *   n_blocks: blocks kept by score per row; n_blocks * block >= index_topk, and
 *   the coarse selection's size ceil(init/block) + ceil(local/block) + 1 +
 *   n_blocks <= 2048.
 *   Workspace: lsa_hier_workspace_size(cfg, n_rows, max_len, block, n_blocks).
 * Returns LSA_DENSE when max_len <= index_topk (every row dense).
 */
LSA_API size_t lsa_hier_workspace_size(const lsa_config* cfg, int32_t n_rows, int64_t max_len, int32_t block,
                                       int32_t n_blocks);
LSA_API lsa_status lsa_hier_select(const lsa_config* cfg, int32_t n_rows, int32_t n_seq,
                                   const int32_t* seq_of_row, const int32_t* pos, const lsa_bf16* q_idx,
                                   const float* w, const lsa_bf16* k_idx, const int64_t* k_off,
                                   const lsa_bf16* k_blk, const int64_t* blk_off, int64_t max_len, int32_t block,
                                   int32_t n_blocks, int32_t* idx, int32_t* count, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * Sparse absorbed-latent MLA, decode ([Lite-Sparse] LSA section: at decode
 * the latent rows are gathered by the top-k indices; 架构总览: kv_lora_rank 512,
 * qk_rope_head_dim 64, 32 heads).
 *
 * Row b (one query of sequence b) attends over the latent rows
 * latent[k_off[b] + idx[b, i]], i < count[b]:
 *   x_i = softmax_scale * (q_abs[b,h,:] . latent[., :576])
 *   out[b,h,:] = sum_i softmax(x)_i * latent[., :512];  lse[b,h] = log sum_i exp(x_i)
 * idx == NULL: dense over all L_b = k_off[b+1]-k_off[b] keys (count unused).
 * q_abs bf16 [batch, 32, 576]; latent bf16 [sum L_b, 576]; idx int32
 * [batch, index_topk]; count int32 [batch]; out bf16 [batch, 32, 512];
 * lse fp32 [batch, 32] or NULL. max_len (host) >= every L_b (sizes split-K).
 * Workspace optional (split-K partials): lsa_workspace_size(LSA_OP_MLA_DECODE).
 * Calls that may overlap on the GPU must not share a workspace (true of every
 * MLA entry point).
 */
/*
 * lsa_sparse_mla_decode_topk: the same attention, for idx / count written by
 * lsa_topk, lsa_forward or lsa_hier_select for these rows with this
 * configuration. Every
 * list then starts with the row's index_init_tokens sink columns and
 * index_local_tokens local columns, which the position alone determines
 * ([Lite-Sparse] LSA section: those columns are always selected), and the
 * kernel gathers and attends over them before it waits for the previous kernel
 * in the stream (the top-k); it reads idx and count only after that wait, and
 * writes nothing before it. So q_abs, latent and k_off are read early: they
 * must not be written by the immediately preceding kernel if that kernel lets
 * its dependents start before it has finished (programmatic dependent launch);
 * kernels of this library never write them. A count other than
 * min(L_b, index_topk) sets LSA_DEVERR_COUNT. Arguments otherwise as
 * lsa_sparse_mla_decode; idx must not be NULL.
 */
LSA_API lsa_status lsa_sparse_mla_decode_topk(const lsa_config* cfg, int32_t batch, const lsa_bf16* q_abs,
                                              const lsa_bf16* latent, const int64_t* k_off, const int32_t* idx,
                                              const int32_t* count, int64_t max_len, lsa_bf16* out, float* lse,
                                              void* ws, size_t ws_bytes, void* stream);

LSA_API lsa_status lsa_sparse_mla_decode(const lsa_config* cfg, int32_t batch, const lsa_bf16* q_abs,
                                 const lsa_bf16* latent, const int64_t* k_off, const int32_t* idx,
                                 const int32_t* count, int64_t max_len, lsa_bf16* out, float* lse,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * lsa_sparse_mla_decode_layer: the cfg->cli_factor attention sub-blocks of a
 * layer that share one selection ([Lite-Sparse] LSA section, cross-layer index
 * reuse: the second sub-block reuses the first one's topk_indices; [LSA-2.0]
 * 跨层索引), in one launch. Sub-block z attends with its own queries q_abs[z]
 * over its own latent cache latent[z] (both packed by the same k_off) and
 * writes out[z] / lse[z], exactly as lsa_sparse_mla_decode_topk would for each
 * z; idx / count must come from lsa_topk, lsa_forward or lsa_hier_select
 * (forced columns first), and the same early start before the top-k applies.
 * q_abs, latent, out, lse: HOST arrays of cli_factor DEVICE pointers (lse
 * itself or its entries may be NULL). All sub-blocks' queries must be ready at
 * the call: a model whose second sub-block's query depends on the first one's
 * output calls lsa_sparse_mla_decode_topk once per sub-block instead.
 * Workspace: lsa_workspace_size(LSA_OP_MLA_DECODE_LAYER, batch, batch, max_len).
 */
LSA_API lsa_status lsa_sparse_mla_decode_layer(const lsa_config* cfg, int32_t batch, const lsa_bf16* const* q_abs,
                                               const lsa_bf16* const* latent, const int64_t* k_off,
                                               const int32_t* idx, const int32_t* count, int64_t max_len,
                                               lsa_bf16* const* out, float* const* lse, void* ws, size_t ws_bytes,
                                               void* stream);

/*
 * lsa_mtp_mla_decode: the draft steps of one multi-token-prediction round over
 * one shared index pass ([LSA-2.0] 多token预测模块集成: the method extends to
 * a three-step MTP module for speculative decoding, and all draft steps share
 * a single index pass), in one launch. The page says only that the pass is
 * shared; reading taken: the index pass and top-k ran once, for the first
 * draft step's query of sequence b at position pos[b] (idx / count from
 * lsa_topk / lsa_forward with that pos, forced columns first). Draft step i
 * (0 <= i < n_draft) has its query at position pos[b] + i; the keys
 * pos[b]+1 .. pos[b]+i (the earlier drafts' and its own) are already in the
 * cache, and a query sees its own key, so step i attends over the shared
 * selection plus those i keys:
 *   out[i][b] = attention of q_abs[i][b] over latent[k_off[b] + j],
 *               j in {idx[b, :count[b]]} U {pos[b]+1 .. pos[b]+i}.
 * All steps read the one latent cache `latent` (the MTP module's), packed by
 * k_off; every sequence must hold keys through pos[b] + n_draft - 1 (a step
 * whose keys run past the sequence sets LSA_DEVERR_POS and attends only to the
 * keys present). 1 <= n_draft <= 4. q_abs, out, lse: HOST arrays of n_draft
 * DEVICE pointers (q_abs[i] bf16 [batch, 32, 576], out[i] bf16 [batch, 32,
 * 512], lse[i] fp32 [batch, 32]; lse or its entries may be NULL). pos int32
 * [batch] (device). Workspace: lsa_workspace_size(LSA_OP_MTP_DECODE, batch,
 * batch, max_len).
 */
LSA_API lsa_status lsa_mtp_mla_decode(const lsa_config* cfg, int32_t n_draft, int32_t batch, const int32_t* pos,
                                      const lsa_bf16* const* q_abs, const lsa_bf16* latent, const int64_t* k_off,
                                      const int32_t* idx, const int32_t* count, int64_t max_len,
                                      lsa_bf16* const* out, float* const* lse, void* ws, size_t ws_bytes,
                                      void* stream);

/*
 * Sparse absorbed-latent MLA, prefill ([Lite-Sparse] LSA section: at prefill
 * a sparse boolean mask built from the indices enters attention). Row r
 * attends over {idx[r, i] : i < count[r]}, which is the set that mask keeps,
 * gathered instead of masked; idx == NULL: dense causal over 0..pos[r].
 * One sequence: latent bf16 [n_keys, 576], every pos[r] < n_keys.
 * Shapes otherwise as lsa_sparse_mla_decode, with n_rows query rows.
 */
LSA_API lsa_status lsa_sparse_mla_prefill(const lsa_config* cfg, int32_t n_rows, const int32_t* pos,
                                  const lsa_bf16* q_abs, const lsa_bf16* latent, int64_t n_keys,
                                  const int32_t* idx, const int32_t* count, lsa_bf16* out,
                                  float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * LoZA attention ("LongCat-Flash-Thinking-ZigZag架构深度剖析", section
 * "LoZA稀疏注意力机制" / "稀疏模式设计": the attention matrix is split into a
 * Sink region (the start of the sequence), a Recent region (the latest
 * context) and a Chunked region (the middle, processed block by block)). The
 * page gives no sizes; reading taken: a query at position p attends to the keys
 * j <= p with j < sink, or p - j < recent, or j / chunk == p / chunk (its own
 * chunk). The set is static, no indexer runs, and attention over it is the same
 * absorbed MLA as lsa_sparse_mla_decode / _prefill (scale, layouts, outputs).
 *
 * mode 0 = decode: row r is a query of sequence seq_of_row[r] (NULL: r) at
 *          position pos[r] (pos NULL: the sequence's last key); latent packed
 *          by k_off like lsa_sparse_mla_decode; max_len >= every sequence's length.
 * mode 1 = prefill: one sequence, latent bf16 [max_len, 576], k_off and
 *          seq_of_row NULL, pos required (every pos[r] < max_len).
 * q_abs bf16 [n_rows, 32, 576], out bf16 [n_rows, 32, 512], lse fp32
 * [n_rows, 32] or NULL. Workspace optional (split-K partials), sized by
 * lsa_workspace_size(LSA_OP_MLA_DECODE) (mode 0) or (LSA_OP_MLA_PREFILL)
 * (mode 1) with the same n_rows and max_len. LSA_ERR_INVALID for a NULL
 * pattern, sink < 0, recent < 0 or chunk < 1. A position outside its sequence
 * sets LSA_DEVERR_POS and is clamped into it; a seq_of_row entry outside
 * [0, n_seq) sets LSA_DEVERR_SEQ and that row attends to nothing (zero output).
 */
typedef struct lsa_loza_pattern {
  int32_t sink;    /* keys at the start every query sees */
  int32_t recent;  /* the query's latest keys, its own included */
  int32_t chunk;   /* the query also sees every earlier key of its chunk [p/chunk*chunk, p] */
} lsa_loza_pattern;
LSA_API lsa_status lsa_loza_mla(const lsa_config* cfg, const lsa_loza_pattern* pattern, int32_t mode, int32_t n_rows,
                                int32_t n_seq, const int32_t* seq_of_row, const int32_t* pos, const int64_t* k_off,
                                int64_t max_len, const lsa_bf16* q_abs, const lsa_bf16* latent, lsa_bf16* out,
                                float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * The whole layer: one index pass and top-k, then cli_factor attention
 * sub-blocks over the same selection ([Lite-Sparse] LSA section, cross-layer
 * index reuse: only the first sub-block owns an indexer; [LSA-2.0] 跨层索引).
 * When max_len <= index_topk the indexer is not run and every sub-block is
 * dense MLA, as the pages' fallback does.
 *
 * mode 0 = decode (rows are queries of sequences given by seq_of_row/k_off;
 *          seq_of_row NULL means row b is the query of sequence b;
 *          each sub-block's latent cache is packed like k_idx);
 * mode 1 = prefill (one sequence, k_off NULL; max_len = keys in the caches).
 * q_abs, latent, out, lse: HOST arrays of cli_factor DEVICE pointers
 *   (lse entries may be NULL; lse itself may be NULL).
 * idx_out int32 [n_rows, index_topk] and count_out int32 [n_rows]: optional
 *   (NULL = keep the selection in the workspace). Unwritten when dense.
 * Workspace: lsa_workspace_size(LSA_OP_FORWARD_*); prefill rows are processed
 * in blocks that fit.
 */
LSA_API lsa_status lsa_forward(const lsa_config* cfg, int32_t mode, int32_t n_rows, int32_t n_seq,
                       const int32_t* seq_of_row, const int32_t* pos, int64_t max_len,
                       const lsa_bf16* q_idx, const float* w, const lsa_bf16* k_idx,
                       const int64_t* k_off, const lsa_bf16* const* q_abs,
                       const lsa_bf16* const* latent, lsa_bf16* const* out, float* const* lse,
                       int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                       void* stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
LSA_API const char* lsa_last_error(void);

/* Synchronising: waits for the current device, returns and clears the sticky
 * device-side flags (LSA_DEVERR_*) in *flags. LSA_ERR_DEVICE if any was set. */
LSA_API lsa_status lsa_device_error(int32_t* flags);

/* Number of kernels this library has launched in the process so far (host
 * counter, no CUDA call). Used to count the launches inside a timed region. */
LSA_API int64_t lsa_launch_count(void);

/*
 * Test hook for the bounded waits of the sparse-MLA kernel (no counterpart in
 * the pages; never needed in normal use). Arms the next sparse-MLA launch made
 * by this host thread, and only that one: every CTA's producer stops handing
 * key tiles to the ring before tile drop_tile (-1: it does not stop), and the
 * attention warps give up any wait after wait_ns nanoseconds (0: the normal
 * 2 s). A wait for a tile that was never issued then runs out: the kernel
 * returns with garbage output for those rows, sets LSA_DEVERR_TIMEOUT, and
 * every copy it did issue has landed before it exits, so the device stays
 * usable. Tests use it to exercise the timeout report.
 */
LSA_API void lsa_debug_arm_mla_wait_test(int64_t wait_ns, int32_t drop_tile);

/* ABI version of this header (1). */
LSA_API int32_t lsa_abi_version(void);

/*
 * Synthetic inputs (tests and benchmarks; not part of the attention path).
 * Counter-based SplitMix64 (Steele, Lea, Flood, OOPSLA 2014): the stream of
 * tensor `tid` under `seed` starts at key = mix64(seed ^ tid*0xD1B54A32D192ED03)
 * and element i is mix64(key + (i+1)*0x9E3779B97F4A7C15). Normal element i is
 * (sum of the eight 16-bit fields of stream elements 2i and 2i+1 - 262140)
 * * fp32(sigma/sqrt(2*(2^32-1)/3)), one fp32 multiply (tails at about 4.9
 * sigma); bf16 outputs round to nearest even. Elements
 * first .. first+n-1 are written to dst[0 .. n-1].
 * lsa_synth_rms_rows_bf16 draws n_rows rows of d values, rounds them to bf16,
 * divides each row by sqrt(sum x^2 / d + 1e-6) in fp64, then rounds to fp32
 * and to bf16 (row first_row+i of the stream goes to dst row i).
 */
LSA_API lsa_status lsa_synth_normal_bf16(lsa_bf16* dst, int64_t n, uint64_t seed, uint64_t tid,
                                 int64_t first, double sigma, void* stream);
LSA_API lsa_status lsa_synth_normal_f32(float* dst, int64_t n, uint64_t seed, uint64_t tid, int64_t first,
                                double sigma, void* stream);
LSA_API lsa_status lsa_synth_rms_rows_bf16(lsa_bf16* dst, int64_t n_rows, int32_t d, uint64_t seed,
                                   uint64_t tid, int64_t first_row, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
