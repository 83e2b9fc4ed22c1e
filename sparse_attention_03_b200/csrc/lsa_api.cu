// C-ABI of liblsa.so: argument checks, workspace carving and kernel dispatch.
// The operations themselves are defined (with their sources) in include/lsa.h.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace lsa {

static thread_local char g_msg[1024];
__device__ int g_dev_err;

lsa_status set_error(lsa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

static std::atomic<int64_t> g_launches{0};
void count_launches(int64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int* device_error_word() {
  static int* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_err) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

lsa_status check_cfg(const lsa_config* c, const char* fn) {
  if (!c) return set_error(LSA_ERR_INVALID, "%s: cfg is NULL", fn);
  if (c->index_n_heads != kHi || c->index_head_dim != kDi || c->n_heads != kH ||
      c->kv_lora_rank != kDV || c->qk_rope_head_dim != kDLat - kDV)
    return set_error(LSA_ERR_UNSUPPORTED,
                     "%s: kernels implement index heads 32x128 and MLA 32 heads x (512+64) only", fn);
  if (c->cli_factor < 1 || c->cli_factor > 2)
    return set_error(LSA_ERR_UNSUPPORTED, "%s: cli_factor must be 1 or 2", fn);
  if (c->index_topk < 1 || c->index_topk > kMaxTopk || c->index_init_tokens < 0 ||
      c->index_local_tokens < 0 ||
      (int64_t)c->index_init_tokens + c->index_local_tokens >= c->index_topk)
    return set_error(LSA_ERR_UNSUPPORTED,
                     "%s: need 0 <= init, 0 <= local, init + local < topk <= 2048", fn);
  if (!(c->softmax_scale > 0.f) || !isfinite(c->softmax_scale))
    return set_error(LSA_ERR_INVALID, "%s: softmax_scale must be finite and > 0", fn);
  return LSA_OK;
}

namespace {

constexpr size_t kAlign = 256;
constexpr int kTopkPreferredRows = 4096;
constexpr size_t kPrefillScoreBudget = size_t(4) << 30;  // bytes of scores per prefill block

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


lsa_status cuda_status(cudaError_t e, const char* fn) {
  if (e == cudaSuccess) return LSA_OK;
  return set_error(LSA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
}

// The top-k's workspace. Rows taken by several CTAs each also get room for the
// threshold bin's candidates beyond the kTopkCap of the base layout: a sixteenth
// of the row (at most 2^18), so that the bin rarely outgrows it.
size_t topk_ws(int n_rows, int64_t max_len = 0) {
  size_t per = kTopkRowBytes;
  if (max_len > 0 && topk_uses_workspace(n_rows, max_len)) {
    const int64_t room = std::min<int64_t>(max_len / 16, int64_t(1) << 18);
    if (room > kTopkCap) per += (size_t)(room - kTopkCap) * sizeof(uint64_t);
  }
  return (size_t)std::min(n_rows, kTopkPreferredRows) * per + kAlign;
}

// Split-K workspace of the MLA launch, whichever split count it picks.
size_t mla_ws(int n_rows, int n_sub, int64_t max_list) {
  return std::max(mla_ws_bytes(n_rows, n_sub, mla_choose_splits(n_rows, n_sub, max_list, false)),
                  mla_ws_bytes(n_rows, n_sub, mla_choose_splits(n_rows, n_sub, max_list, true)));
}

// Workspace of one forward block of R rows (sparse path).
size_t forward_block_ws(const lsa_config* c, int R, int64_t max_len) {
  return align_up((size_t)R * max_len * sizeof(float)) + align_up((size_t)R * kTopkHistStride * sizeof(uint32_t)) +
         align_up((size_t)R * c->index_topk * sizeof(int32_t)) +
         align_up((size_t)R * sizeof(int32_t)) + topk_ws(R, max_len) + mla_ws(R, c->cli_factor, c->index_topk);
}

int prefill_block_rows(int n_rows, int64_t max_len) {
  int64_t r = (int64_t)(kPrefillScoreBudget / ((size_t)max_len * sizeof(float)));
  r = std::max<int64_t>(64, r / 64 * 64);
  return (int)std::min<int64_t>(r, n_rows);
}

lsa_status run_index_scores(const lsa_config* c, int n_rows, int n_seq, const int32_t* seq_of_row,
                            int seq_identity, const int32_t* pos, const lsa_bf16* q_idx, const float* w,
                            const lsa_bf16* k_idx, const int64_t* k_off, int64_t max_len,
                            float* scores, int64_t ld, cudaStream_t st, uint32_t* topk_hist = nullptr) {
  IndexArgs a;
  a.q_idx = q_idx;
  a.w = w;
  a.k_idx = k_idx;
  a.k_off = k_off;
  a.seq_of_row = seq_of_row;
  a.seq_identity = seq_identity;
  a.pos = pos;
  a.n_rows = n_rows;
  a.n_seq = n_seq;
  a.max_len = max_len;
  a.n_init = c->index_init_tokens;
  a.n_loc = c->index_local_tokens;
  a.scores = scores;
  a.ld = ld;
  a.err = device_error_word();
  if (topk_hist) {
    const lsa_status s0 = cuda_status(
        launch_zero_words(topk_hist, (size_t)n_rows * kTopkHistStride, st), "lsa_index_scores");
    if (s0 != LSA_OK) return s0;
  }
  if (!index_prefill_supported(a))
    return cuda_status(launch_index_decode(a, st, topk_hist, c->index_topk), "lsa_index_scores");
  lsa_status s1 = cuda_status(launch_index_prefill(a, st), "lsa_index_scores");
  if (s1 != LSA_OK || !topk_hist) return s1;
  // The tensor-core epilogue has no room for per-row histograms: one pass over
  // the fresh scores builds them instead.
  TopkArgs t;
  t.scores = scores;
  t.ld = ld;
  t.pos = pos;
  t.n_rows = n_rows;
  t.max_len = max_len;
  t.topk = c->index_topk;
  t.n_init = c->index_init_tokens;
  t.n_loc = c->index_local_tokens;
  t.idx = nullptr;
  t.count = nullptr;
  t.ws = nullptr;
  t.ws_bytes = 0;
  return cuda_status(launch_topk_hist_only(t, topk_hist, st), "lsa_index_scores");
}

lsa_status run_topk(const lsa_config* c, int n_rows, const int32_t* pos, int64_t max_len,
                    const float* scores, int64_t ld, int32_t* idx, int32_t* count, void* ws,
                    size_t ws_bytes, cudaStream_t st, uint32_t* hist_ext = nullptr) {
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.pos = pos;
  a.n_rows = n_rows;
  a.max_len = max_len;
  a.topk = c->index_topk;
  a.n_init = c->index_init_tokens;
  a.n_loc = c->index_local_tokens;
  a.idx = idx;
  a.count = count;
  a.hist_ext = hist_ext;
  uintptr_t p = (reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~uintptr_t(kAlign - 1);
  a.ws = reinterpret_cast<void*>(p);
  const size_t slack = ws ? p - reinterpret_cast<uintptr_t>(ws) : 0;
  a.ws_bytes = ws_bytes > slack ? ws_bytes - slack : 0;
  if (max_len > c->index_topk && topk_uses_workspace(n_rows, max_len) && a.ws_bytes < kTopkRowBytes)
    return set_error(LSA_ERR_WORKSPACE, "lsa_topk: workspace below one row (%zu bytes)",
                     (size_t)kTopkRowBytes);
  const lsa_status st2 = cuda_status(launch_topk(a, st), "lsa_topk");
  if (st2 != LSA_OK) return st2;
  return max_len <= c->index_topk ? LSA_DENSE : LSA_OK;
}

MlaArgs mla_args(const lsa_config* c, int n_sub, int n_rows, int decode) {
  MlaArgs a = {};
  a.n_rows = n_rows;
  a.n_sub = n_sub;
  a.decode = decode;
  a.topk = c->index_topk;
  a.scale = c->softmax_scale;
  a.err = device_error_word();
  return a;
}


// Hierarchical selection: the block-level constants and the workspace layout.
struct HierPlan {
  int n_init_b, n_loc_b, kb;  // forced sink / recent blocks, blocks kept per row
  int64_t nb_max, ld_b, ld_c; // blocks per row at most, coarse and compact row strides
  size_t off_pos_c, off_hist, off_coarse, off_kept, off_kept_n, off_sorted, off_cand, off_topk, total;
};

HierPlan hier_plan(const lsa_config* c, int n_rows, int64_t max_len, int block, int n_blocks) {
  HierPlan h;
  h.n_init_b = (c->index_init_tokens + block - 1) / block;
  h.n_loc_b = (c->index_local_tokens + block - 1) / block + 1;
  h.kb = h.n_init_b + h.n_loc_b + n_blocks;
  h.nb_max = (max_len + block - 1) / block;
  h.ld_b = (h.nb_max + 3) / 4 * 4;
  h.ld_c = (int64_t)h.kb * block;
  const size_t R = (size_t)n_rows;
  size_t o = 0;
  h.off_pos_c = o;  o += align_up(R * 4);
  h.off_hist = o;   o += align_up(R * kTopkHistStride * 4);
  h.off_coarse = o; o += align_up(R * h.ld_b * 4);
  h.off_kept = o;   o += align_up(R * h.kb * 4);
  h.off_kept_n = o; o += align_up(R * 4);
  h.off_sorted = o; o += align_up(R * h.kb * 4);
  h.off_cand = o;   o += align_up(R * h.ld_c * 4);
  h.off_topk = o;   o += topk_ws(n_rows);
  h.total = o + kAlign;
  return h;
}

lsa_status check_hier(const lsa_config* c, int block, int n_blocks, const char* fn) {
  if (block < 16 || block > 1024 || block % 16 != 0)
    return set_error(LSA_ERR_UNSUPPORTED, "%s: block must be a multiple of 16 in [16, 1024]", fn);
  if (n_blocks < 1 || (int64_t)n_blocks * block < c->index_topk)
    return set_error(LSA_ERR_UNSUPPORTED, "%s: need n_blocks >= 1 and n_blocks * block >= index_topk", fn);
  const int64_t kb = (int64_t)(c->index_init_tokens + block - 1) / block +
                     (c->index_local_tokens + block - 1) / block + 1 + n_blocks;
  if (kb > 2048) return set_error(LSA_ERR_UNSUPPORTED, "%s: the coarse selection exceeds 2048 blocks", fn);
  return LSA_OK;
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" {

int32_t lsa_abi_version(void) { return 1; }

int64_t lsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* lsa_last_error(void) { return g_msg; }

void lsa_config_default(lsa_config* c) {
  if (!c) return;
  c->index_n_heads = 32;
  c->index_head_dim = 128;
  c->index_topk = 2048;
  c->index_init_tokens = 16;
  c->index_local_tokens = 1024;
  c->cli_factor = 2;
  c->n_heads = 32;
  c->kv_lora_rank = 512;
  c->qk_rope_head_dim = 64;
  c->softmax_scale = (float)(1.0 / sqrt(128.0 + 64.0));
}

size_t lsa_workspace_size(const lsa_config* c, int32_t op, int32_t n_rows, int32_t n_seq,
                          int64_t max_len) {
  (void)n_seq;
  if (check_cfg(c, "lsa_workspace_size") != LSA_OK || n_rows < 0 || max_len < 1) return 0;
  if (n_rows == 0) return kAlign;
  const int64_t list = std::min<int64_t>(max_len, c->index_topk);
  switch (op) {
    case LSA_OP_TOPK:
      return max_len <= c->index_topk ? kAlign : topk_ws(n_rows, max_len);
    case LSA_OP_MLA_DECODE:
    case LSA_OP_MLA_PREFILL:
      return std::max(mla_ws(n_rows, 1, max_len), mla_ws(n_rows, 1, list)) + kAlign;
    case LSA_OP_FORWARD_DECODE:
      if (max_len <= c->index_topk) return mla_ws(n_rows, c->cli_factor, max_len) + kAlign;
      return forward_block_ws(c, n_rows, max_len) + kAlign;
    case LSA_OP_FORWARD_PREFILL:
      if (max_len <= c->index_topk) return mla_ws(n_rows, c->cli_factor, max_len) + kAlign;
      return forward_block_ws(c, prefill_block_rows(n_rows, max_len), max_len) + kAlign;
    case LSA_OP_INDEX_PROJECT:
      return project_ws_bytes(n_rows) + kAlign;
    case LSA_OP_MLA_DECODE_LAYER:
      return mla_ws(n_rows, c->cli_factor, list) + kAlign;
    case LSA_OP_MTP_DECODE:
      return mla_ws(n_rows, kMaxSub, list) + kAlign;
    default:
      return 0;
  }
}

lsa_status lsa_device_error(int32_t* flags) {
  int* p = device_error_word();
  if (!p) return set_error(LSA_ERR_CUDA, "lsa_device_error: no device error word");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "lsa_device_error");
  int v = 0;
  e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e, "lsa_device_error");
  if (flags) *flags = v;
  if (v) return set_error(LSA_ERR_DEVICE, "lsa_device_error: device flags 0x%x", v);
  return LSA_OK;
}

lsa_status lsa_index_scores(const lsa_config* c, int32_t n_rows, int32_t n_seq,
                            const int32_t* seq_of_row, const int32_t* pos, const lsa_bf16* q_idx,
                            const float* w, const lsa_bf16* k_idx, const int64_t* k_off,
                            int64_t max_len, float* scores, int64_t ld, uint32_t* topk_hist,
                            void* stream) {
  const char* fn = "lsa_index_scores";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (n_rows < 0 || n_seq < 1 || max_len < 1 || ld < max_len)
    return set_error(LSA_ERR_INVALID, "%s: need n_rows >= 0, n_seq >= 1, 1 <= max_len <= ld", fn);
  if (!k_off && n_seq != 1) return set_error(LSA_ERR_INVALID, "%s: k_off is NULL with n_seq > 1", fn);
  if (n_rows == 0) return LSA_OK;
  if (!pos || !q_idx || !w || !k_idx || !scores)
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (!aligned16(q_idx) || !aligned16(k_idx))
    return set_error(LSA_ERR_INVALID, "%s: q_idx and k_idx must be 16-byte aligned", fn);
  if (topk_hist && !aligned16(topk_hist))
    return set_error(LSA_ERR_INVALID, "%s: topk_hist must be 16-byte aligned", fn);
  return run_index_scores(c, n_rows, n_seq, seq_of_row, 0, pos, q_idx, w, k_idx, k_off, max_len,
                          scores, ld, (cudaStream_t)stream, topk_hist);
}

lsa_status lsa_topk(const lsa_config* c, int32_t n_rows, const int32_t* pos, int64_t max_len,
                    const float* scores, int64_t ld, uint32_t* topk_hist, int32_t* idx,
                    int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  const char* fn = "lsa_topk";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (n_rows < 0 || max_len < 1 || ld < max_len)
    return set_error(LSA_ERR_INVALID, "%s: need n_rows >= 0 and 1 <= max_len <= ld", fn);
  if (n_rows == 0) return max_len <= c->index_topk ? LSA_DENSE : LSA_OK;
  if (!pos || !scores || !idx || !count) return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (topk_hist && !aligned16(topk_hist))
    return set_error(LSA_ERR_INVALID, "%s: topk_hist must be 16-byte aligned", fn);
  if (max_len > c->index_topk && !ws && topk_uses_workspace(n_rows, max_len))
    return set_error(LSA_ERR_WORKSPACE, "%s: workspace is NULL", fn);
  return run_topk(c, n_rows, pos, max_len, scores, ld, idx, count, ws, ws_bytes, (cudaStream_t)stream,
                  topk_hist);
}

lsa_status lsa_index_project(const lsa_config* c, int32_t n_rows, int32_t n_seq, const int32_t* seq_of_row,
                             const int32_t* pos, const int64_t* k_off, int64_t max_len, const lsa_bf16* c_q,
                             const lsa_bf16* hidden, const lsa_bf16* wq_b, const lsa_bf16* wk,
                             const lsa_bf16* wproj, const lsa_bf16* k_norm_w, int32_t q_lora_rank,
                             int32_t hidden_size, float rope_theta, lsa_bf16* q_idx, float* w, lsa_bf16* k_cache,
                             void* ws, size_t ws_bytes, void* stream) {
  const char* fn = "lsa_index_project";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (n_rows < 0 || n_seq < 1 || max_len < 1)
    return set_error(LSA_ERR_INVALID, "%s: need n_rows >= 0, n_seq >= 1, max_len >= 1", fn);
  if (q_lora_rank <= 0 || q_lora_rank % 32 || hidden_size <= 0 || hidden_size % 32)
    return set_error(LSA_ERR_INVALID, "%s: q_lora_rank and hidden_size must be positive multiples of 32", fn);
  if (!(rope_theta > 1.f)) return set_error(LSA_ERR_INVALID, "%s: rope_theta must exceed 1", fn);
  if (n_rows == 0) return LSA_OK;
  if (!pos || !c_q || !hidden || !wq_b || !wk || !wproj || !k_norm_w || !q_idx || !w || !k_cache)
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (n_seq > 1 && !k_off) return set_error(LSA_ERR_INVALID, "%s: several sequences need k_off", fn);
  const void* al[] = {c_q, hidden, wq_b, wk, wproj, k_norm_w, q_idx, w, k_cache};
  for (const void* p : al)
    if (!aligned16(p)) return set_error(LSA_ERR_INVALID, "%s: arrays must be 16-byte aligned", fn);
  if (!ws || ws_bytes < project_ws_bytes(n_rows))
    return set_error(LSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed", fn, project_ws_bytes(n_rows));
  if ((n_rows + 63) / 64 > 65535) return set_error(LSA_ERR_UNSUPPORTED, "%s: at most 4194240 rows", fn);
  ProjectLaunch L;
  L.c_q = reinterpret_cast<const uint16_t*>(c_q);
  L.hidden = reinterpret_cast<const uint16_t*>(hidden);
  L.wq_b = reinterpret_cast<const uint16_t*>(wq_b);
  L.wk = reinterpret_cast<const uint16_t*>(wk);
  L.wproj = reinterpret_cast<const uint16_t*>(wproj);
  L.k_norm_w = reinterpret_cast<const uint16_t*>(k_norm_w);
  L.seq_of_row = seq_of_row;
  L.pos = pos;
  L.k_off = k_off;
  L.n_rows = n_rows;
  L.n_seq = n_seq;
  L.q_lora = q_lora_rank;
  L.hidden_dim = hidden_size;
  L.max_len = max_len;
  L.theta = rope_theta;
  L.q_out = reinterpret_cast<uint16_t*>(q_idx);
  L.w_out = w;
  L.k_cache = reinterpret_cast<uint16_t*>(k_cache);
  L.ws = ws;
  L.err = device_error_word();
  return cuda_status(launch_index_project(L, (cudaStream_t)stream), fn);
}

}  // extern "C"

namespace {
lsa_status mla_decode(const char* fn, bool lists_from_topk, const lsa_config* c, int32_t batch,
                      const lsa_bf16* q_abs, const lsa_bf16* latent, const int64_t* k_off, const int32_t* idx,
                      const int32_t* count, int64_t max_len, lsa_bf16* out, float* lse, void* ws, size_t ws_bytes,
                      void* stream) {
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (batch < 0 || max_len < 1) return set_error(LSA_ERR_INVALID, "%s: need batch >= 0, max_len >= 1", fn);
  if (batch == 0) return LSA_OK;
  if (!q_abs || !latent || !k_off || !out || (idx && !count))
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (!aligned16(q_abs) || !aligned16(latent) || !aligned16(out))
    return set_error(LSA_ERR_INVALID, "%s: q_abs, latent and out must be 16-byte aligned", fn);
  MlaArgs a = mla_args(c, 1, batch, 1);
  a.q[0] = q_abs;
  a.lat[0] = latent;
  a.out[0] = out;
  a.lse[0] = lse;
  a.k_off = k_off;
  a.n_seq = batch;
  a.idx = idx;
  a.count = count;
  a.max_list = idx ? c->index_topk : max_len;
  a.ws = ws;
  a.ws_bytes = ws ? ws_bytes : 0;
  if (lists_from_topk) {
    if (!idx) return set_error(LSA_ERR_INVALID, "%s: idx is NULL", fn);
    a.forced_first = 1;
    a.n_init = c->index_init_tokens;
    a.n_loc = c->index_local_tokens;
  }
  return cuda_status(launch_mla(a, (cudaStream_t)stream), fn);
}
}  // namespace

extern "C" {

lsa_status lsa_sparse_mla_decode(const lsa_config* c, int32_t batch, const lsa_bf16* q_abs,
                                 const lsa_bf16* latent, const int64_t* k_off, const int32_t* idx,
                                 const int32_t* count, int64_t max_len, lsa_bf16* out, float* lse,
                                 void* ws, size_t ws_bytes, void* stream) {
  return mla_decode("lsa_sparse_mla_decode", false, c, batch, q_abs, latent, k_off, idx, count, max_len, out, lse,
                    ws, ws_bytes, stream);
}

lsa_status lsa_sparse_mla_decode_topk(const lsa_config* c, int32_t batch, const lsa_bf16* q_abs,
                                      const lsa_bf16* latent, const int64_t* k_off, const int32_t* idx,
                                      const int32_t* count, int64_t max_len, lsa_bf16* out, float* lse,
                                      void* ws, size_t ws_bytes, void* stream) {
  return mla_decode("lsa_sparse_mla_decode_topk", true, c, batch, q_abs, latent, k_off, idx, count, max_len, out,
                    lse, ws, ws_bytes, stream);
}

}  // extern "C"

namespace {
// Sub-blocks over one shared forced-first selection in one launch: the
// cli_factor sub-blocks of a layer (mtp 0), or the draft steps of an MTP round
// (mtp 1: step z also sees keys pos+1 .. pos+z).
lsa_status mla_decode_shared(const char* fn, const lsa_config* c, int n_sub, int mtp, int32_t batch,
                             const int32_t* pos, const lsa_bf16* const* q_abs, const lsa_bf16* const* latent,
                             const int64_t* k_off, const int32_t* idx, const int32_t* count, int64_t max_len,
                             lsa_bf16* const* out, float* const* lse, void* ws, size_t ws_bytes, void* stream) {
  if (batch < 0 || max_len < 1) return set_error(LSA_ERR_INVALID, "%s: need batch >= 0, max_len >= 1", fn);
  if (batch == 0) return LSA_OK;
  if (!q_abs || !latent || !out || !k_off || !idx || !count || (mtp && !pos))
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  MlaArgs a = mla_args(c, n_sub, batch, 1);
  for (int z = 0; z < n_sub; ++z) {
    const lsa_bf16* lat = latent[mtp ? 0 : z];
    if (!q_abs[z] || !lat || !out[z]) return set_error(LSA_ERR_INVALID, "%s: NULL pointer for sub-block %d", fn, z);
    if (!aligned16(q_abs[z]) || !aligned16(lat) || !aligned16(out[z]))
      return set_error(LSA_ERR_INVALID, "%s: q_abs, latent and out must be 16-byte aligned", fn);
    a.q[z] = q_abs[z];
    a.lat[z] = lat;
    a.out[z] = out[z];
    a.lse[z] = lse ? lse[z] : nullptr;
  }
  a.k_off = k_off;
  a.n_seq = batch;
  a.pos = pos;
  a.idx = idx;
  a.count = count;
  a.max_list = c->index_topk;
  a.forced_first = 1;
  a.n_init = c->index_init_tokens;
  a.n_loc = c->index_local_tokens;
  a.mtp = mtp;
  a.ws = ws;
  a.ws_bytes = ws ? ws_bytes : 0;
  return cuda_status(launch_mla(a, (cudaStream_t)stream), fn);
}
}  // namespace

extern "C" {

lsa_status lsa_sparse_mla_decode_layer(const lsa_config* c, int32_t batch, const lsa_bf16* const* q_abs,
                                       const lsa_bf16* const* latent, const int64_t* k_off, const int32_t* idx,
                                       const int32_t* count, int64_t max_len, lsa_bf16* const* out,
                                       float* const* lse, void* ws, size_t ws_bytes, void* stream) {
  const char* fn = "lsa_sparse_mla_decode_layer";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  return mla_decode_shared(fn, c, c->cli_factor, 0, batch, nullptr, q_abs, latent, k_off, idx, count, max_len, out,
                           lse, ws, ws_bytes, stream);
}

lsa_status lsa_mtp_mla_decode(const lsa_config* c, int32_t n_draft, int32_t batch, const int32_t* pos,
                              const lsa_bf16* const* q_abs, const lsa_bf16* latent, const int64_t* k_off,
                              const int32_t* idx, const int32_t* count, int64_t max_len, lsa_bf16* const* out,
                              float* const* lse, void* ws, size_t ws_bytes, void* stream) {
  const char* fn = "lsa_mtp_mla_decode";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (n_draft < 1 || n_draft > kMaxSub)
    return set_error(LSA_ERR_UNSUPPORTED, "%s: n_draft must be in [1, %d]", fn, kMaxSub);
  const lsa_bf16* lat[kMaxSub] = {latent};
  return mla_decode_shared(fn, c, n_draft, 1, batch, pos, q_abs, lat, k_off, idx, count, max_len, out, lse, ws,
                           ws_bytes, stream);
}

void lsa_debug_arm_mla_wait_test(int64_t wait_ns, int32_t drop_tile) {
  mla_arm_wait_test((long long)wait_ns, (int)drop_tile);
}

lsa_status lsa_sparse_mla_prefill(const lsa_config* c, int32_t n_rows, const int32_t* pos,
                                  const lsa_bf16* q_abs, const lsa_bf16* latent, int64_t n_keys,
                                  const int32_t* idx, const int32_t* count, lsa_bf16* out,
                                  float* lse, void* ws, size_t ws_bytes, void* stream) {
  const char* fn = "lsa_sparse_mla_prefill";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (n_rows < 0 || n_keys < 1) return set_error(LSA_ERR_INVALID, "%s: need n_rows >= 0, n_keys >= 1", fn);
  if (n_rows == 0) return LSA_OK;
  if (!pos || !q_abs || !latent || !out || (idx && !count))
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (!aligned16(q_abs) || !aligned16(latent) || !aligned16(out))
    return set_error(LSA_ERR_INVALID, "%s: q_abs, latent and out must be 16-byte aligned", fn);
  MlaArgs a = mla_args(c, 1, n_rows, 0);
  a.q[0] = q_abs;
  a.lat[0] = latent;
  a.out[0] = out;
  a.lse[0] = lse;
  a.pos = pos;
  a.n_keys = n_keys;
  a.idx = idx;
  a.count = count;
  a.max_list = idx ? c->index_topk : n_keys;
  a.ws = ws;
  a.ws_bytes = ws ? ws_bytes : 0;
  return cuda_status(launch_mla(a, (cudaStream_t)stream), fn);
}

lsa_status lsa_loza_mla(const lsa_config* c, const lsa_loza_pattern* pat, int32_t mode, int32_t n_rows,
                        int32_t n_seq, const int32_t* seq_of_row, const int32_t* pos, const int64_t* k_off,
                        int64_t max_len, const lsa_bf16* q_abs, const lsa_bf16* latent, lsa_bf16* out, float* lse,
                        void* ws, size_t ws_bytes, void* stream) {
  const char* fn = "lsa_loza_mla";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (!pat) return set_error(LSA_ERR_INVALID, "%s: pattern is NULL", fn);
  if (pat->sink < 0 || pat->recent < 0 || pat->chunk < 1)
    return set_error(LSA_ERR_INVALID, "%s: need sink >= 0, recent >= 0, chunk >= 1", fn);
  if ((mode != 0 && mode != 1) || n_rows < 0 || n_seq < 1 || max_len < 1)
    return set_error(LSA_ERR_INVALID, "%s: need mode 0/1, n_rows >= 0, n_seq >= 1, max_len >= 1", fn);
  if (mode == 0 && !k_off) return set_error(LSA_ERR_INVALID, "%s: decode needs k_off", fn);
  if (mode == 1 && (n_seq != 1 || k_off || seq_of_row))
    return set_error(LSA_ERR_INVALID, "%s: prefill takes one sequence (k_off and seq_of_row NULL)", fn);
  if (n_rows == 0) return LSA_OK;
  if ((mode == 1 && !pos) || !q_abs || !latent || !out) return set_error(LSA_ERR_INVALID, "%s: NULL argument", fn);
  if (!aligned16(q_abs) || !aligned16(latent) || !aligned16(out))
    return set_error(LSA_ERR_INVALID, "%s: q_abs, latent and out must be 16-byte aligned", fn);
  MlaArgs a = mla_args(c, 1, n_rows, mode == 0 ? 1 : 0);
  a.q[0] = q_abs;
  a.lat[0] = latent;
  a.out[0] = out;
  a.lse[0] = lse;
  a.k_off = mode == 0 ? k_off : nullptr;
  a.seq_of_row = mode == 0 ? seq_of_row : nullptr;
  a.n_seq = n_seq;
  a.pos = pos;
  a.n_keys = max_len;
  a.idx = nullptr;
  a.count = nullptr;
  a.loza = 1;
  a.loza_sink = pat->sink;
  a.loza_recent = pat->recent;
  a.loza_chunk = pat->chunk;
  // a row's set: at most the sink plus the longer of its window and its chunk
  a.max_list = std::min<int64_t>(max_len, (int64_t)pat->sink + std::max<int64_t>(pat->recent, pat->chunk));
  a.ws = ws;
  a.ws_bytes = ws ? ws_bytes : 0;
  return cuda_status(launch_mla(a, (cudaStream_t)stream), fn);
}

lsa_status lsa_forward(const lsa_config* c, int32_t mode, int32_t n_rows, int32_t n_seq,
                       const int32_t* seq_of_row, const int32_t* pos, int64_t max_len,
                       const lsa_bf16* q_idx, const float* w, const lsa_bf16* k_idx,
                       const int64_t* k_off, const lsa_bf16* const* q_abs,
                       const lsa_bf16* const* latent, lsa_bf16* const* out, float* const* lse,
                       int32_t* idx_out, int32_t* count_out, void* ws, size_t ws_bytes,
                       void* stream) {
  const char* fn = "lsa_forward";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  const cudaStream_t st = (cudaStream_t)stream;
  const int cli = c->cli_factor;
  if ((mode != 0 && mode != 1) || n_rows < 0 || n_seq < 1 || max_len < 1)
    return set_error(LSA_ERR_INVALID, "%s: need mode 0/1, n_rows >= 0, n_seq >= 1, max_len >= 1", fn);
  if (mode == 0 && !k_off) return set_error(LSA_ERR_INVALID, "%s: decode needs k_off", fn);
  if (mode == 1 && n_seq != 1) return set_error(LSA_ERR_INVALID, "%s: prefill takes one sequence", fn);
  if (n_rows == 0) return LSA_OK;
  if (!pos || !q_abs || !latent || !out) return set_error(LSA_ERR_INVALID, "%s: NULL argument", fn);
  for (int z = 0; z < cli; ++z) {
    if (!q_abs[z] || !latent[z] || !out[z])
      return set_error(LSA_ERR_INVALID, "%s: NULL sub-block pointer %d", fn, z);
    if (!aligned16(q_abs[z]) || !aligned16(latent[z]) || !aligned16(out[z]))
      return set_error(LSA_ERR_INVALID, "%s: sub-block %d arrays must be 16-byte aligned", fn, z);
  }
  const bool dense = max_len <= c->index_topk;
  if (!dense) {
    if (!q_idx || !w || !k_idx) return set_error(LSA_ERR_INVALID, "%s: NULL indexer argument", fn);
    if (!aligned16(q_idx) || !aligned16(k_idx))
      return set_error(LSA_ERR_INVALID, "%s: q_idx and k_idx must be 16-byte aligned", fn);
    if (!ws) return set_error(LSA_ERR_WORKSPACE, "%s: workspace is NULL", fn);
  }

  // Carve the workspace.
  uintptr_t base = (reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~uintptr_t(kAlign - 1);
  size_t avail = ws ? ws_bytes - std::min(ws_bytes, (size_t)(base - reinterpret_cast<uintptr_t>(ws))) : 0;

  MlaArgs m = mla_args(c, cli, n_rows, mode == 0 ? 1 : 0);
  for (int z = 0; z < cli; ++z) {
    m.q[z] = q_abs[z];
    m.lat[z] = latent[z];
    m.out[z] = out[z];
    m.lse[z] = lse ? lse[z] : nullptr;
  }
  m.k_off = mode == 0 ? k_off : nullptr;
  m.seq_of_row = mode == 0 ? seq_of_row : nullptr;
  m.n_seq = n_seq;
  m.pos = pos;
  m.n_keys = max_len;

  if (dense) {
    // The pages' fallback: no index pass, dense MLA in every sub-block.
    m.idx = nullptr;
    m.count = nullptr;
    m.max_list = max_len;
    m.ws = reinterpret_cast<void*>(base);
    m.ws_bytes = avail;
    return cuda_status(launch_mla(m, st), fn);
  }

  int R = n_rows;
  if (mode == 1) R = prefill_block_rows(n_rows, max_len);
  while (R > 1 && forward_block_ws(c, R, max_len) > avail) R = R > 64 ? R / 64 * 32 : R / 2;
  if (forward_block_ws(c, R, max_len) > avail)
    return set_error(LSA_ERR_WORKSPACE, "%s: workspace %zu below the minimum %zu", fn, ws_bytes,
                     forward_block_ws(c, 1, max_len) + kAlign);
  if (mode == 0 && R < n_rows)
    return set_error(LSA_ERR_WORKSPACE, "%s: decode needs lsa_workspace_size(LSA_OP_FORWARD_DECODE)", fn);

  char* p = reinterpret_cast<char*>(base);
  float* scores = reinterpret_cast<float*>(p);
  p += align_up((size_t)R * max_len * sizeof(float));
  uint32_t* hist_ws = reinterpret_cast<uint32_t*>(p);
  p += align_up((size_t)R * kTopkHistStride * sizeof(uint32_t));
  int32_t* idx_ws = reinterpret_cast<int32_t*>(p);
  p += align_up((size_t)R * c->index_topk * sizeof(int32_t));
  int32_t* cnt_ws = reinterpret_cast<int32_t*>(p);
  p += align_up((size_t)R * sizeof(int32_t));
  void* topk_w = p;  // 256-byte aligned (every region above is a multiple of 256)
  const size_t topk_bytes = topk_ws(R, max_len);
  p += topk_bytes;
  // Decode: the indexer builds the top-k's histogram while the scores are in
  // registers, which saves the top-k one pass over the scores and one launch;
  // not for rows short enough that the top-k holds all their scores anyway
  // (there it would only add the histogram's zeroing launch).
  const bool fuse_hist =
      mode == 0 && max_len - c->index_init_tokens - c->index_local_tokens > kTopkShortMid;
  void* mla_w = p;
  const size_t mla_bytes = mla_ws(R, cli, c->index_topk);

  for (int r0 = 0; r0 < n_rows; r0 += R) {
    const int nr = std::min(R, n_rows - r0);
    int32_t* idx_b = idx_out ? idx_out + (int64_t)r0 * c->index_topk : idx_ws;
    int32_t* cnt_b = count_out ? count_out + r0 : cnt_ws;
    uint32_t* hist = fuse_hist ? hist_ws : nullptr;
    s = run_index_scores(c, nr, n_seq, seq_of_row ? seq_of_row + r0 : nullptr, mode == 0, pos + r0,
                         q_idx + (int64_t)r0 * kHi * kDi, w + (int64_t)r0 * kHi, k_idx, k_off,
                         max_len, scores, max_len, st, hist);
    if (s != LSA_OK) return s;
    s = run_topk(c, nr, pos + r0, max_len, scores, max_len, idx_b, cnt_b, topk_w, topk_bytes, st, hist);
    if (s != LSA_OK && s != LSA_DENSE) return s;
    MlaArgs b = m;
    b.n_rows = nr;
    for (int z = 0; z < cli; ++z) {
      b.q[z] = q_abs[z] + (int64_t)r0 * kH * kDLat;
      b.out[z] = out[z] + (int64_t)r0 * kH * kDV;
      b.lse[z] = m.lse[z] ? m.lse[z] + (int64_t)r0 * kH : nullptr;
    }
    if (b.seq_of_row) b.seq_of_row += r0;
    else if (mode == 0 && r0 > 0) return set_error(LSA_ERR_INVALID, "%s: internal row split", fn);
    b.pos = pos + r0;
    b.idx = idx_b;
    b.count = cnt_b;
    // the lists come from the top-k just above: the forced columns lead them
    b.forced_first = 1;
    b.n_init = c->index_init_tokens;
    b.n_loc = c->index_local_tokens;
    b.max_list = c->index_topk;
    b.ws = mla_w;
    b.ws_bytes = mla_bytes;
    s = cuda_status(launch_mla(b, st), fn);
    if (s != LSA_OK) return s;
  }
  return LSA_OK;
}


lsa_status lsa_block_summaries(const lsa_config* c, int32_t n_items, int32_t n_seq, const int32_t* item_seq,
                               const int32_t* item_blk, const lsa_bf16* k_idx, const int64_t* k_off,
                               const int64_t* blk_off, int32_t block, lsa_bf16* k_blk, void* stream) {
  const char* fn = "lsa_block_summaries";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  if (block < 16 || block > 1024 || block % 16 != 0)
    return set_error(LSA_ERR_UNSUPPORTED, "%s: block must be a multiple of 16 in [16, 1024]", fn);
  if (n_items < 0 || n_seq < 1) return set_error(LSA_ERR_INVALID, "%s: need n_items >= 0 and n_seq >= 1", fn);
  if (n_items == 0) return LSA_OK;
  if (!item_seq || !item_blk || !k_idx || !k_off || !blk_off || !k_blk)
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (!aligned16(k_idx) || !aligned16(k_blk))
    return set_error(LSA_ERR_INVALID, "%s: k_idx and k_blk must be 16-byte aligned", fn);
  BlockSumArgs a;
  a.k_idx = k_idx;
  a.k_off = k_off;
  a.blk_off = blk_off;
  a.item_seq = item_seq;
  a.item_blk = item_blk;
  a.n_items = n_items;
  a.n_seq = n_seq;
  a.block = block;
  a.k_blk = k_blk;
  a.err = device_error_word();
  return cuda_status(launch_block_summaries(a, (cudaStream_t)stream), fn);
}

size_t lsa_hier_workspace_size(const lsa_config* c, int32_t n_rows, int64_t max_len, int32_t block,
                               int32_t n_blocks) {
  if (check_cfg(c, "lsa_hier_workspace_size") != LSA_OK || n_rows < 0 || max_len < 1 ||
      check_hier(c, block, n_blocks, "lsa_hier_workspace_size") != LSA_OK)
    return 0;
  if (n_rows == 0) return kAlign;
  return hier_plan(c, n_rows, max_len, block, n_blocks).total;
}

lsa_status lsa_hier_select(const lsa_config* c, int32_t n_rows, int32_t n_seq, const int32_t* seq_of_row,
                           const int32_t* pos, const lsa_bf16* q_idx, const float* w, const lsa_bf16* k_idx,
                           const int64_t* k_off, const lsa_bf16* k_blk, const int64_t* blk_off, int64_t max_len,
                           int32_t block, int32_t n_blocks, int32_t* idx, int32_t* count, void* ws,
                           size_t ws_bytes, void* stream) {
  const char* fn = "lsa_hier_select";
  lsa_status s = check_cfg(c, fn);
  if (s != LSA_OK) return s;
  s = check_hier(c, block, n_blocks, fn);
  if (s != LSA_OK) return s;
  if (n_rows < 0 || n_seq < 1 || max_len < 1)
    return set_error(LSA_ERR_INVALID, "%s: need n_rows >= 0, n_seq >= 1, max_len >= 1", fn);
  if ((!k_off || !blk_off) && n_seq != 1)
    return set_error(LSA_ERR_INVALID, "%s: k_off / blk_off NULL with n_seq > 1", fn);
  if (!k_off || !blk_off) return set_error(LSA_ERR_INVALID, "%s: k_off and blk_off are required", fn);
  if (n_rows == 0) return max_len <= c->index_topk ? LSA_DENSE : LSA_OK;
  if (!pos || !q_idx || !w || !k_idx || !k_blk || !idx || !count)
    return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(k_blk))
    return set_error(LSA_ERR_INVALID, "%s: q_idx, k_idx and k_blk must be 16-byte aligned", fn);
  cudaStream_t st = (cudaStream_t)stream;
  const HierPlan h = hier_plan(c, n_rows, max_len, block, n_blocks);
  if (!ws || ws_bytes < h.total)
    return set_error(LSA_ERR_WORKSPACE, "%s: workspace %zu below %zu", fn, ws_bytes, h.total);
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + kAlign - 1) & ~uintptr_t(kAlign - 1));
  int32_t* pos_c = reinterpret_cast<int32_t*>(base + h.off_pos_c);
  float* coarse = reinterpret_cast<float*>(base + h.off_coarse);
  int32_t* kept = reinterpret_cast<int32_t*>(base + h.off_kept);
  int32_t* kept_n = reinterpret_cast<int32_t*>(base + h.off_kept_n);
  int32_t* sorted = reinterpret_cast<int32_t*>(base + h.off_sorted);
  float* cand = reinterpret_cast<float*>(base + h.off_cand);
  uint32_t* hist_c = reinterpret_cast<uint32_t*>(base + h.off_hist);
  void* topk_w = base + h.off_topk;
  const size_t topk_bytes = topk_ws(n_rows);

  // the flat top-k's arguments over this call's rows (a per-call view of the workspace)
  auto topk_args = [&](const float* scores, int64_t ld, int64_t len, int topk, int n_init, int n_loc, int32_t* out,
                       int32_t* cnt) {
    TopkArgs t;
    t.scores = scores;
    t.ld = ld;
    t.pos = pos;
    t.n_rows = n_rows;
    t.max_len = len;
    t.topk = topk;
    t.n_init = n_init;
    t.n_loc = n_loc;
    t.idx = out;
    t.count = cnt;
    t.ws = topk_w;
    t.ws_bytes = topk_bytes;
    return t;
  };
  if (max_len <= c->index_topk) {  // every row dense: 0 .. pos, nothing to score
    const TopkArgs t = topk_args(coarse, h.ld_b, max_len, c->index_topk, c->index_init_tokens,
                                 c->index_local_tokens, idx, count);
    s = cuda_status(launch_topk(t, st), fn);
    return s == LSA_OK ? LSA_DENSE : s;
  }
  // coarse stage: the indexer over the summaries and the flat top-k one level up,
  // both reading each row's position divided by the block size
  IndexArgs a;
  a.q_idx = q_idx;
  a.w = w;
  a.k_idx = k_blk;
  a.k_off = blk_off;
  a.seq_of_row = seq_of_row;
  a.seq_identity = 0;
  a.pos = pos;
  a.pos_div = block;
  a.n_rows = n_rows;
  a.n_seq = n_seq;
  a.max_len = h.nb_max;
  a.n_init = h.n_init_b;
  a.n_loc = h.n_loc_b;
  a.scores = coarse;
  a.ld = h.ld_b;
  a.err = device_error_word();
  s = cuda_status(launch_index_decode(a, st), fn);
  if (s != LSA_OK) return s;
  TopkArgs tb = topk_args(coarse, h.ld_b, h.nb_max, h.kb, h.n_init_b, h.n_loc_b, kept, kept_n);
  tb.pos_div = block;
  tb.zero_hist = hist_c;  // for the fine stage, which builds the compact rows' histograms
  s = cuda_status(launch_topk(tb, st), fn);
  if (s != LSA_OK) return s;
  // fine stage: the kept blocks' tokens into compact rows, then the flat top-k
  // over them, writing token columns
  HierFineArgs f;
  f.ix = a;
  f.ix.k_idx = k_idx;
  f.ix.k_off = k_off;
  f.ix.pos_div = 1;
  f.ix.max_len = max_len;
  f.ix.n_init = c->index_init_tokens;
  f.ix.n_loc = c->index_local_tokens;
  f.ix.scores = nullptr;
  f.kept = kept;
  f.kept_n = kept_n;
  f.kb = h.kb;
  f.block = block;
  f.nb_max = h.nb_max;
  f.sorted = sorted;
  f.pos_c = pos_c;
  f.topk = c->index_topk;
  f.cand = cand;
  f.ld_c = h.ld_c;
  f.hist = hist_c;
  s = cuda_status(launch_hier_fine(f, st), fn);
  if (s != LSA_OK) return s;
  TopkArgs tc = topk_args(cand, h.ld_c, h.ld_c, c->index_topk, c->index_init_tokens, c->index_local_tokens, idx,
                          count);
  tc.pos = pos_c;
  tc.hist_ext = hist_c;
  tc.col_map = sorted;
  tc.col_block = block;
  tc.col_ld = h.kb;
  return cuda_status(launch_topk(tc, st), fn);
}

}  // extern "C"
