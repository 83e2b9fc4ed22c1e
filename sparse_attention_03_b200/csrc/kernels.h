// Internal launchers of the LSA kernels (host side). Not part of the C-ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "lsa.h"

namespace lsa {

// Records the message for lsa_last_error() and returns `st`.
lsa_status set_error(lsa_status st, const char* fmt, ...);
// Address of this device's sticky error word (device memory).
int* device_error_word();
// Adds n to the process-wide launch counter (lsa_launch_count).
void count_launches(int64_t n);
// LSA_OK when the configuration is one the kernels implement; otherwise the
// status (with its message recorded for lsa_last_error) naming the function.
lsa_status check_cfg(const lsa_config* c, const char* fn);

struct IndexArgs {
  const uint16_t* q_idx;   // [n_rows, 32, 128]
  const float* w;          // [n_rows, 32]
  const uint16_t* k_idx;   // packed [sum L, 128]
  const int64_t* k_off;    // [n_seq+1] or null
  const int32_t* seq_of_row;  // null: sequence r (seq_identity) or sequence 0
  int seq_identity;
  const int32_t* pos;
  int pos_div = 1;          // the row's position is pos[r] / pos_div (-1 when pos[r] < 0)
  int n_rows, n_seq;
  int64_t max_len;
  int n_init, n_loc;
  float* scores;
  int64_t ld;
  int* err;
};

// Streaming indexer: each CTA scores a run of keys of one row (decode shape).
// With hist != null it also adds, for rows with more than `topk` visible keys,
// the top 11 bits of every middle-column score key into hist (per row,
// kTopkHistStride words apart, zeroed by the caller): the top-k's first pass.
cudaError_t launch_index_decode(const IndexArgs& a, cudaStream_t st, uint32_t* hist = nullptr,
                                int topk = 0);
// Tensor-core indexer for many rows of one sequence (prefill shape).
bool index_prefill_supported(const IndexArgs& a);
cudaError_t launch_index_prefill(const IndexArgs& a, cudaStream_t st);

struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* pos;
  int pos_div = 1;          // as IndexArgs::pos_div
  int n_rows;
  int64_t max_len;
  int topk, n_init, n_loc;
  int32_t* idx;
  int32_t* count;
  void* ws;
  size_t ws_bytes;
  // Per-row histograms built by the indexer (kTopkHistStride words apart), or
  // null: the top-k then builds them itself. The multi-CTA select keeps its
  // per-row counters in the 8 words after each row's bins (zero on entry, as the
  // indexer leaves them; the row's last CTA zeroes them again).
  uint32_t* hist_ext = nullptr;
  // Optional map from column j to the emitted index: col_map[r * col_ld + j /
  // col_block] * col_block + j % col_block (compact rows of whole blocks). With a
  // map every row goes through the one-CTA-per-row kernel.
  const int32_t* col_map = nullptr;
  int col_block = 1;
  int64_t col_ld = 0;      // <= 2048
  // Optional: rows of another histogram buffer (kTopkHistStride words apart) that
  // this call clears, row r by row r's CTA, for a later producer. Also forces
  // the one-CTA-per-row kernel.
  uint32_t* zero_hist = nullptr;
};
constexpr int kTopkCap = 4096;                              // candidates per row: the base layout, and shared memory
constexpr size_t kTopkRowBytes = 2048 * 4 + 32 + kTopkCap * 8;  // hist + ctl + candidates
constexpr int kTopkHistStride = 2048 + 8;                   // words between rows' histograms
// Rows with at most this many middle columns are "short" for the one-CTA
// top-k: every score sits in registers, so a histogram built elsewhere saves
// that kernel nothing.
constexpr int64_t kTopkShortMid = 8192;

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st);
// Clears n_words 32-bit words on the stream with a kernel (keeps the launch chain).
cudaError_t launch_zero_words(void* p, size_t n_words, cudaStream_t st);
bool topk_uses_workspace(int n_rows, int64_t max_len);
// Fills hist (rows kTopkHistStride words apart, zeroed by the caller) from scores.
cudaError_t launch_topk_hist_only(const TopkArgs& a, uint32_t* hist, cudaStream_t st);
cudaError_t launch_topk_dense(const TopkArgs& a, cudaStream_t st);

// The indexer's own projections and the key-cache append (upstream of the path).
struct ProjectLaunch {
  const uint16_t* c_q;      // [n_rows, q_lora] bf16
  const uint16_t* hidden;   // [n_rows, hidden_dim] bf16
  const uint16_t* wq_b;     // [32 * 128, q_lora] bf16
  const uint16_t* wk;       // [128, hidden_dim] bf16
  const uint16_t* wproj;    // [32, hidden_dim] bf16
  const uint16_t* k_norm_w; // [128] bf16
  const int32_t* seq_of_row;
  const int32_t* pos;
  const int64_t* k_off;
  int n_rows, n_seq, q_lora, hidden_dim;
  int64_t max_len;
  double theta;
  uint16_t* q_out;
  float* w_out;
  uint16_t* k_cache;
  void* ws;
  int* err;
};
size_t project_ws_bytes(int n_rows);
cudaError_t launch_index_project(const ProjectLaunch& L, cudaStream_t st);

constexpr int kMaxSub = 4;  // sub-blocks (or MTP draft steps) of one MLA launch
struct MlaArgs {
  // Per sub-block z < n_sub (grid z): its queries, latent cache, outputs.
  const uint16_t* q[kMaxSub];
  const uint16_t* lat[kMaxSub];
  uint16_t* out[kMaxSub];
  float* lse[kMaxSub];
  const int64_t* k_off;      // decode: [n_seq+1]
  const int32_t* seq_of_row; // decode: row -> sequence (null: identity)
  const int32_t* pos;        // prefill: required; decode: optional (null: the whole sequence)
  const int32_t* idx;        // [n_rows, topk] or null (dense)
  const int32_t* count;
  int n_rows, n_seq, topk, decode, n_sub;
  // The index lists were written by the top-k for these rows (every non-dense
  // row's list starts with its n_init sink and n_loc local columns): the kernel
  // attends over those before it waits for the previous kernel in the stream.
  int forced_first = 0, n_init = 0, n_loc = 0;
  // MTP draft steps (forced-first lists only): sub-block z is draft step z,
  // whose query sits z positions after the index owner's; it attends over the
  // shared list and also over the keys pos+1 .. pos+z.
  int mtp = 0;
  // LoZA rows (no index list): each row attends to keys [0, loza_sink) and to
  // the run from the earlier of its recent window's and its chunk's first key
  // up to its own position.
  int loza = 0, loza_sink = 0, loza_recent = 0, loza_chunk = 1;
  int64_t n_keys;            // prefill: rows in latent
  int64_t max_list;          // host bound on keys per row (sizes split-K)
  float scale;
  void* ws;
  size_t ws_bytes;
  int* err;
  // Bounded waits: the math warps give up a wait after wait_ns. Test hook:
  // drop_tile >= 0 makes every CTA's producer stop before that tile, so the
  // wait for it runs out (the timeout report path); -1 in normal use.
  long long wait_ns = 2000000000ll;
  int drop_tile = -1;
};
// Split-K workspace bytes (partials and merge tickets) for a given split count.
size_t mla_ws_bytes(int n_rows, int n_sub, int n_split);
int mla_choose_splits(int n_rows, int n_sub, int64_t max_list, bool forced_first = false);
// Arms the next launch_mla on this host thread with the test hook above.
void mla_arm_wait_test(long long wait_ns, int drop_tile);
cudaError_t launch_mla(const MlaArgs& a, cudaStream_t st);

}  // namespace lsa

namespace lsa {

// Hierarchical indexing: block summaries, and the pieces of the two-stage
// selection that are not the flat indexer and top-k themselves.
struct BlockSumArgs {
  const uint16_t* k_idx;   // packed [sum L, 128] bf16
  const int64_t* k_off;    // [n_seq+1]
  const int64_t* blk_off;  // [n_seq+1]
  const int32_t* item_seq;
  const int32_t* item_blk;
  int n_items, n_seq, block;
  uint16_t* k_blk;         // packed [sum ceil(L/block), 128] bf16
  int* err;
};
cudaError_t launch_block_summaries(const BlockSumArgs& a, cudaStream_t st);


struct HierFineArgs {
  IndexArgs ix;             // token-level rows, keys and forcing (scores unused)
  const int32_t* kept;      // [n_rows, kb] kept blocks, unordered
  const int32_t* kept_n;    // [n_rows]
  int kb, block;
  int64_t nb_max;           // blocks a row can have (bounds the kept ids)
  int32_t* sorted;          // out [n_rows, kb]: the kept blocks in ascending order
  int32_t* pos_c;           // out [n_rows]: the compact slot of the row's own token (see hier_fine_kernel)
  int topk;
  float* cand;              // out [n_rows, ld_c]: slot i = token sorted[i / block] * block + i % block
  int64_t ld_c;
  uint32_t* hist;           // out: the compact rows' top-k histograms (kTopkHistStride apart, zeroed)
};
// Scores the tokens of each row's kept blocks into the compact rows.
cudaError_t launch_hier_fine(const HierFineArgs& a, cudaStream_t st);


}  // namespace lsa
