// Top-k with forced sink/local columns and the dense fallback.
//
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）": keep the index_topk columns of
// highest score; the index_init_tokens sink and index_local_tokens local
// columns are +inf and so always kept; when the cached length is at most
// index_topk the indexer yields nothing and attention is dense.
//
// Design. The forced columns are emitted by formula, never sorted. The rest of
// the budget (k_rem = topk - init - local) is chosen among the middle columns
// [init, n - local) by a radix select on the order-preserving uint32 image of
// the fp32 score, extended with the bit-inverted column index so that every
// value is unique and ties go to the lower index. Three kernels per row block:
//   1. histogram of the top 11 key bits (many CTAs per row, shared-memory
//      counts flushed with global atomics);
//   2. every CTA finds the threshold bin from the histogram, emits columns in
//      higher bins straight to the output and appends columns in the threshold
//      bin to a per-row candidate buffer;
//   3. one CTA per row finishes the select on the candidates (the remaining 21
//      key bits and 32 index bits, 11 bits per pass, stopping as soon as a bin
//      holds exactly what is still needed), writes the forced columns, the
//      count, and handles dense rows. If the candidate buffer overflowed (many
//      equal scores), it rescans the row instead.
// No kernel waits on another CTA; kernel boundaries order the passes.
#include "common.cuh"
#include "kernels.h"

namespace lsa {
namespace {

constexpr int kBins = 2048;
constexpr int kHistThreads = 256;
constexpr int kResolveThreads = 512;
constexpr int64_t kChunk = 16384;
constexpr uint64_t kLow53 = (1ull << 53) - 1;

// Per-row workspace: a zeroed histogram/control block, then the candidates.
struct HistCtl {
  uint32_t hist[kBins];
  uint32_t ctl[8];  // 0: emitted above, 1: candidates, 2: threshold bin, 3: count above it
};
static_assert(sizeof(HistCtl) + kTopkCap * sizeof(uint64_t) == kTopkRowBytes, "workspace layout");

struct RowGeom {
  int64_t n, lo, hi;  // visible columns; middle range [lo, hi)
  bool dense;
};

__device__ __forceinline__ RowGeom row_geom(const TopkArgs& a, int r) {
  RowGeom g;
  g.n = (int64_t)a.pos[r] + 1;
  if (g.n < 0) g.n = 0;
  if (g.n > a.max_len) g.n = a.max_len;
  g.dense = g.n <= a.topk;
  g.lo = a.n_init;
  g.hi = g.n - a.n_loc;
  return g;
}

// For a histogram h[0..2048) and a budget `need`, finds the bin d such that
// (count in bins above d) < need <= (count in bins >= d). Block-wide; every
// thread returns the same answer.
template <int THREADS>
__device__ void find_threshold(const uint32_t* h, uint32_t need, int& bin_out,
                               uint32_t& above_out, int* s_bin, uint32_t* s_above,
                               uint32_t* s_warp) {
  constexpr int PER = kBins / THREADS;
  constexpr int WARPS = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    *s_bin = 0;
    *s_above = 0;
  }
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) mine += h[tid * PER + i];
  // inclusive suffix sum within the warp
  uint32_t v = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, v, off);
    if (lane + off < 32) v += y;
  }
  if (lane == 0) s_warp[warp] = v;  // warp total
  __syncthreads();
  uint32_t warp_above = 0;
  for (int w2 = warp + 1; w2 < WARPS; ++w2) warp_above += s_warp[w2];
  const uint32_t above = v - mine + warp_above;  // count in bins of higher threads
  if (above < need && above + mine >= need) {
    uint32_t cum = above;
    for (int b = tid * PER + PER - 1; b >= tid * PER; --b) {
      if (cum + h[b] >= need) {
        *s_bin = b;
        *s_above = cum;
        break;
      }
      cum += h[b];
    }
  }
  __syncthreads();
  bin_out = *s_bin;
  above_out = *s_above;
  __syncthreads();
}

__global__ void __launch_bounds__(kHistThreads)
    topk_hist_kernel(TopkArgs a, int row0, HistCtl* hc) {
  __shared__ uint32_t h[kBins];
  const int r = row0 + blockIdx.y;
  const RowGeom g = row_geom(a, r);
  if (g.dense) return;
  const int64_t s = g.lo + (int64_t)blockIdx.x * kChunk;
  const int64_t e = min(s + kChunk, g.hi);
  if (s >= e) return;
  for (int i = threadIdx.x; i < kBins; i += kHistThreads) h[i] = 0;
  __syncthreads();
  const float* __restrict__ srow = a.scores + (int64_t)r * a.ld;
  for (int64_t j = s + threadIdx.x; j < e; j += kHistThreads)
    atomicAdd(&h[score_key(srow[j]) >> 21], 1u);
  __syncthreads();
  HistCtl& w = hc[blockIdx.y];
  for (int i = threadIdx.x; i < kBins; i += kHistThreads)
    if (h[i]) atomicAdd(&w.hist[i], h[i]);
}

__global__ void __launch_bounds__(kHistThreads)
    topk_collect_kernel(TopkArgs a, int row0, HistCtl* hc, uint64_t* cand_all) {
  __shared__ uint32_t h[kBins];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_warp[kHistThreads / 32];
  const int r = row0 + blockIdx.y;
  const RowGeom g = row_geom(a, r);
  if (g.dense) return;
  const int64_t s = g.lo + (int64_t)blockIdx.x * kChunk;
  const int64_t e = min(s + kChunk, g.hi);
  if (s >= e) return;
  HistCtl& w = hc[blockIdx.y];
  uint64_t* __restrict__ cand = cand_all + (int64_t)blockIdx.y * kTopkCap;
  for (int i = threadIdx.x; i < kBins; i += kHistThreads) h[i] = w.hist[i];
  __syncthreads();
  const uint32_t k_rem = (uint32_t)(a.topk - a.n_init - a.n_loc);
  int bin;
  uint32_t above;
  find_threshold<kHistThreads>(h, k_rem, bin, above, &s_bin, &s_above, s_warp);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    w.ctl[2] = (uint32_t)bin;
    w.ctl[3] = above;
  }
  const float* __restrict__ srow = a.scores + (int64_t)r * a.ld;
  int32_t* __restrict__ out = a.idx + (int64_t)r * a.topk + a.n_init + a.n_loc;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t base = s + warp * 32; base < e; base += kHistThreads) {
    const int64_t j = base + lane;
    uint32_t key = 0;
    int kb = -1;
    if (j < e) {
      key = score_key(srow[j]);
      kb = (int)(key >> 21);
    }
    const uint32_t up = __ballot_sync(0xffffffffu, kb > bin);
    const uint32_t eq = __ballot_sync(0xffffffffu, kb == bin);
    if (up) {
      uint32_t slot0 = 0;
      if (lane == 0) slot0 = atomicAdd(&w.ctl[0], (uint32_t)__popc(up));
      slot0 = __shfl_sync(0xffffffffu, slot0, 0);
      const uint32_t slot = slot0 + __popc(up & ((1u << lane) - 1u));
      if (kb > bin && slot < k_rem) out[slot] = (int32_t)j;
    }
    if (eq) {
      uint32_t slot0 = 0;
      if (lane == 0) slot0 = atomicAdd(&w.ctl[1], (uint32_t)__popc(eq));
      slot0 = __shfl_sync(0xffffffffu, slot0, 0);
      const uint32_t slot = slot0 + __popc(eq & ((1u << lane) - 1u));
      if (kb == bin && slot < (uint32_t)kTopkCap)
        cand[slot] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
    }
  }
}

__global__ void __launch_bounds__(kResolveThreads)
    topk_resolve_kernel(TopkArgs a, int row0, const HistCtl* hc, const uint64_t* cand_all) {
  __shared__ uint32_t h[kBins];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_warp[kResolveThreads / 32], s_slot;
  const int r = row0 + blockIdx.x;
  const RowGeom g = row_geom(a, r);
  int32_t* __restrict__ out = a.idx + (int64_t)r * a.topk;
  const int tid = threadIdx.x;
  if (g.dense) {
    for (int i = tid; i < a.topk; i += kResolveThreads) out[i] = (i < g.n) ? i : -1;
    if (tid == 0) a.count[r] = (int32_t)g.n;
    return;
  }
  for (int i = tid; i < a.n_init; i += kResolveThreads) out[i] = i;
  for (int i = tid; i < a.n_loc; i += kResolveThreads) out[a.n_init + i] = (int32_t)(g.hi + i);
  if (tid == 0) a.count[r] = a.topk;

  const HistCtl& w = hc[blockIdx.x];
  const uint64_t* __restrict__ cand = cand_all + (int64_t)blockIdx.x * kTopkCap;
  const uint32_t bin0 = w.ctl[2];
  const uint32_t above0 = w.ctl[3];
  const uint32_t n_cand = w.ctl[1];
  const bool use_cand = n_cand <= (uint32_t)kTopkCap;
  const uint32_t k_rem = (uint32_t)(a.topk - a.n_init - a.n_loc);
  uint32_t need = k_rem - above0;
  const uint32_t need0 = need;
  const float* __restrict__ srow = a.scores + (int64_t)r * a.ld;

  // Calls f(v53, column) for every element of the threshold bin.
  auto for_each = [&](auto&& f) {
    if (use_cand) {
      for (uint32_t i = tid; i < n_cand; i += kResolveThreads) {
        const uint64_t c = cand[i];
        f(c & kLow53, (int64_t)(0xFFFFFFFFu - (uint32_t)c));
      }
    } else {
      for (int64_t j = g.lo + tid; j < g.hi; j += kResolveThreads) {
        const uint32_t key = score_key(srow[j]);
        if ((key >> 21) == bin0) {
          const uint64_t c = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
          f(c & kLow53, j);
        }
      }
    }
  };

  uint64_t prefix = 0;
  int decided = 0;  // bits of v53 fixed so far, from the top
  const int widths[5] = {11, 11, 11, 11, 9};
  for (int lvl = 0; lvl < 5; ++lvl) {
    const int wdt = widths[lvl];
    const int shift = 53 - decided - wdt;
    for (int i = tid; i < kBins; i += kResolveThreads) h[i] = 0;
    __syncthreads();
    for_each([&](uint64_t v, int64_t) {
      if ((v >> (53 - decided)) == prefix)
        atomicAdd(&h[(uint32_t)(v >> shift) & ((1u << wdt) - 1u)], 1u);
    });
    __syncthreads();
    int d;
    uint32_t above;
    find_threshold<kResolveThreads>(h, need, d, above, &s_bin, &s_above, s_warp);
    const uint32_t cnt = h[d];
    need -= above;
    prefix = (prefix << wdt) | (uint64_t)d;
    decided += wdt;
    __syncthreads();
    if (cnt == need) break;  // the whole bin is taken
  }
  if (tid == 0) s_slot = 0;
  __syncthreads();
  int32_t* __restrict__ dst = out + a.n_init + a.n_loc + above0;
  const int sh = 53 - decided;
  for_each([&](uint64_t v, int64_t j) {
    if ((v >> sh) >= prefix) {
      const uint32_t slot = atomicAdd(&s_slot, 1u);
      if (slot < need0) dst[slot] = (int32_t)j;
    }
  });
}

}  // namespace

cudaError_t launch_topk_dense(const TopkArgs& a, cudaStream_t st) {
  for (int row0 = 0; row0 < a.n_rows; row0 += 65535) {
    const int nr = min(65535, a.n_rows - row0);
    topk_resolve_kernel<<<nr, kResolveThreads, 0, st>>>(a, row0, nullptr, nullptr);
    count_launches(1);
  }
  return cudaGetLastError();
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
  if (a.n_rows <= 0) return cudaSuccess;
  if (a.max_len <= a.topk) return launch_topk_dense(a, st);
  const int64_t rows_fit = (int64_t)(a.ws_bytes / kTopkRowBytes);
  const int blk = (int)min64(min64(rows_fit, a.n_rows), 65535);
  const int64_t chunks = (a.max_len + kChunk - 1) / kChunk;
  HistCtl* hc = static_cast<HistCtl*>(a.ws);
  uint64_t* cand = reinterpret_cast<uint64_t*>(hc + blk);
  for (int row0 = 0; row0 < a.n_rows; row0 += blk) {
    const int nr = min(blk, a.n_rows - row0);
    cudaError_t e = cudaMemsetAsync(hc, 0, (size_t)nr * sizeof(HistCtl), st);
    if (e != cudaSuccess) return e;
    topk_hist_kernel<<<dim3((unsigned)chunks, (unsigned)nr), kHistThreads, 0, st>>>(a, row0, hc);
    topk_collect_kernel<<<dim3((unsigned)chunks, (unsigned)nr), kHistThreads, 0, st>>>(a, row0, hc, cand);
    topk_resolve_kernel<<<nr, kResolveThreads, 0, st>>>(a, row0, hc, cand);
    count_launches(3);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace lsa
