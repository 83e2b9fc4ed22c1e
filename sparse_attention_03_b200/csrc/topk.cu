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
// value is unique and ties go to the lower index. The first pass is a histogram
// of the top 11 key bits, built by the decode indexer while the scores are in
// registers, or here. Two kernel shapes:
//   * many or short rows: one CTA per row does everything, with the
//     threshold-bin candidates in shared memory. A short row's scores sit in
//     registers; a long row without a histogram (a prefill block) is read once:
//     a sample of the row sets a bound, one pass keeps every score above it in
//     shared memory, and the select finishes there, with the exact two-pass
//     path as the fallback when the bound admits too few or too many;
//   * few long rows: many CTAs per row. Each finds the threshold bin, places
//     its chunk's columns with one block-wide prefix sum and one global atomic,
//     and the last CTA of the row (an atomic ticket) finishes the select on the
//     candidates, which the workspace keeps (up to a sixteenth of the row).
// When the threshold bin holds more candidates than shared memory, the next 11
// key bits split it first (the digits above the threshold digit go straight
// out), over the workspace's candidates or, in the one-CTA kernel, over the row;
// only equal keys beyond that fall back to rescanning the row per level.
// No kernel waits on another CTA.
#include "common.cuh"
#include "kernels.h"
#include "launch.h"
#include "radix.cuh"

namespace lsa {
namespace {

constexpr int kHistThreads = 256;
constexpr int64_t kChunk = 4096;     // scores per CTA in the histogram and collect passes
constexpr int kUnroll = 8;           // loads in flight per lane
constexpr uint64_t kLow53 = (1ull << 53) - 1;

// Per-row workspace: a zeroed histogram/control block, then the candidates.
struct HistCtl {
  uint32_t hist[kBins];
  // 0: emitted above; 4 and 5, one 64-bit counter: the threshold-bin candidates
  // (low word) and the CTAs that have finished (high word), so that the last
  // CTA's ticket also returns the candidate count
  uint32_t ctl[8];
};
static_assert(sizeof(HistCtl) + kTopkCap * sizeof(uint64_t) == kTopkRowBytes, "workspace layout");

struct RowGeom {
  int64_t n, lo, hi;  // visible columns; middle range [lo, hi)
  bool dense;
};

__device__ __forceinline__ RowGeom row_geom(const TopkArgs& a, int r) {
  RowGeom g;
  const int pr = a.pos[r];
  g.n = (int64_t)(a.pos_div == 1 ? pr : (pr >= 0 ? pr / a.pos_div : -1)) + 1;
  if (g.n < 0) g.n = 0;
  if (g.n > a.max_len) g.n = a.max_len;
  g.dense = g.n <= a.topk;
  g.lo = a.n_init;
  g.hi = g.n - a.n_loc;
  return g;
}

__global__ void __launch_bounds__(kHistThreads)
    topk_hist_kernel(TopkArgs a, int row0, HistCtl* hc) {
  __shared__ uint32_t h[kBins];
  pdl_wait();
  pdl_trigger();  // dependents may launch now; they wait for this grid before reading its outputs
  const int r = row0 + blockIdx.y;
  const RowGeom g = row_geom(a, r);
  if (g.dense) return;
  const int64_t s = g.lo + (int64_t)blockIdx.x * kChunk;
  const int64_t e = min(s + kChunk, g.hi);
  if (s >= e) return;
  for (int i = threadIdx.x; i < kBins; i += kHistThreads) h[i] = 0;
  __syncthreads();
  const float* __restrict__ srow = a.scores + (int64_t)r * a.ld;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // each warp takes 32 * kUnroll consecutive scores per round, all loads first
  for (int64_t base = s + warp * 32 * kUnroll; base < e; base += kHistThreads * kUnroll) {
    float v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t j = base + lane + 32 * u;
      v[u] = j < e ? srow[j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (base + lane + 32 * u < e) atomicAdd(&h[score_key(v[u]) >> 21], 1u);
  }
  __syncthreads();
  HistCtl& w = hc[blockIdx.y];
  for (int i = threadIdx.x; i < kBins; i += kHistThreads)
    if (h[i]) atomicAdd(&w.hist[i], h[i]);
}

// Every CTA finds the threshold bin from the row's histogram, then handles its
// chunk with each thread's scores in registers: one block-wide prefix sum places
// every emitted column, and one global atomic per CTA claims the row's slots
// (no per-warp round trips to a shared counter). The last CTA of a row to finish
// (an atomic ticket; nothing waits) selects the rest inside the threshold bin
// from the candidates, staged in shared memory, and writes the forced columns.
constexpr int kPerThread = kChunk / kHistThreads;  // 16 scores per thread
static_assert(kPerThread == 2 * kUnroll, "two rounds of kUnroll loads per thread");

__global__ void __launch_bounds__(kHistThreads, 4)
    topk_select_kernel(TopkArgs a, int row0, HistCtl* hc, uint64_t* cand_all, uint32_t cand_cap) {
  __shared__ uint32_t h[kBins];
  __shared__ uint64_t scand[kTopkCap];
  __shared__ int s_bin, s_last;
  __shared__ uint32_t s_above, s_warp[kHistThreads / 32], s_wu[kHistThreads / 32], s_we[kHistThreads / 32];
  __shared__ uint32_t s_base_u, s_base_e, s_slot, s_ncand;
  pdl_wait();
  pdl_trigger();  // dependents may launch now; they wait for this grid before reading its outputs
  const int r = row0 + blockIdx.y;
  const RowGeom g = row_geom(a, r);
  int32_t* __restrict__ row_out = a.idx + (int64_t)r * a.topk;
  const int tid = threadIdx.x;
  if (g.dense) {
    if (blockIdx.x == 0) {
      for (int i = tid; i < a.topk; i += kHistThreads) row_out[i] = (i < g.n) ? i : -1;
      if (tid == 0) a.count[r] = (int32_t)g.n;
    }
    return;
  }
  const int64_t s = g.lo + (int64_t)blockIdx.x * kChunk;
  const int64_t e = min(s + kChunk, g.hi);
  if (s >= e) return;
  const uint32_t n_chunks = (uint32_t)((g.hi - g.lo + kChunk - 1) / kChunk);
  HistCtl& w = hc[blockIdx.y];
  uint64_t* __restrict__ cand = cand_all + (int64_t)blockIdx.y * cand_cap;
  // This chunk's scores are requested first; the histogram and the threshold
  // search overlap their latency.
  const float* __restrict__ srow = a.scores + (int64_t)r * a.ld;
  const int lane = tid & 31, warp = tid >> 5;
  const int64_t wbase = s + warp * 32 * kUnroll;  // the second round adds kHistThreads * kUnroll
  float sv[kPerThread];
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int64_t j = wbase + (i / kUnroll) * kHistThreads * kUnroll + lane + 32 * (i % kUnroll);
    sv[i] = j < e ? srow[j] : 0.f;
  }
  const uint32_t* hsrc = a.hist_ext ? a.hist_ext + (int64_t)r * kTopkHistStride : w.hist;
  uint32_t* ctl = a.hist_ext ? a.hist_ext + (int64_t)r * kTopkHistStride + kBins : w.ctl;
  for (int i = tid; i < kBins; i += kHistThreads) h[i] = hsrc[i];
  __syncthreads();
  const uint32_t k_rem = (uint32_t)(a.topk - a.n_init - a.n_loc);
  int bin;
  uint32_t above;
  find_threshold<kHistThreads>(h, k_rem, bin, above, &s_bin, &s_above, s_warp);
  // bin of each score; -1 marks positions past the chunk's end
  auto kbin = [&](int i) -> int {
    const int64_t j = wbase + (i / kUnroll) * kHistThreads * kUnroll + lane + 32 * (i % kUnroll);
    return j < e ? (int)(score_key(sv[i]) >> 21) : -1;
  };
  uint32_t nu = 0, ne = 0;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int kb = kbin(i);
    nu += kb > bin;
    ne += kb == bin;
  }
  // exclusive prefix sums over the CTA (warp scans, then the warp totals)
  uint32_t iu = nu, ie = ne;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t yu = __shfl_up_sync(0xffffffffu, iu, off);
    const uint32_t ye = __shfl_up_sync(0xffffffffu, ie, off);
    if (lane >= off) {
      iu += yu;
      ie += ye;
    }
  }
  if (lane == 31) {
    s_wu[warp] = iu;
    s_we[warp] = ie;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t tu = 0, te = 0;
    for (int i = 0; i < kHistThreads / 32; ++i) {
      const uint32_t a_u = s_wu[i], a_e = s_we[i];
      s_wu[i] = tu;
      s_we[i] = te;
      tu += a_u;
      te += a_e;
    }
    s_base_u = tu ? atomicAdd(&ctl[0], tu) : 0u;
    s_base_e = te ? (uint32_t)atomicAdd(reinterpret_cast<unsigned long long*>(&ctl[4]), (unsigned long long)te) : 0u;
  }
  __syncthreads();
  uint32_t ou = s_base_u + s_wu[warp] + iu - nu;
  uint32_t oe = s_base_e + s_we[warp] + ie - ne;
  int32_t* __restrict__ mid = row_out + a.n_init + a.n_loc;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int64_t j = wbase + (i / kUnroll) * kHistThreads * kUnroll + lane + 32 * (i % kUnroll);
    const int kb = kbin(i);
    if (kb > bin) {
      if (ou < k_rem) mid[ou] = (int32_t)j;
      ++ou;
    } else if (kb == bin) {
      if (oe < cand_cap)
        cand[oe] = ((uint64_t)score_key(sv[i]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
      ++oe;
    }
  }

  // ---- the last CTA of the row finishes it ----
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned long long t = atomicAdd(reinterpret_cast<unsigned long long*>(&ctl[4]), 1ull << 32);
    s_last = (uint32_t)(t >> 32) == n_chunks - 1;
    s_ncand = (uint32_t)t;  // every CTA reserved its candidates before its ticket
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = tid; i < a.n_init; i += kHistThreads) row_out[i] = i;
  for (int i = tid; i < a.n_loc; i += kHistThreads) row_out[a.n_init + i] = (int32_t)(g.hi + i);
  if (tid == 0) {
    a.count[r] = a.topk;
    s_slot = 0;
  }
  const uint32_t n_cand = s_ncand;
  const uint32_t need0 = k_rem - above;
  // Where the rest of the select runs: the threshold-bin candidates in shared
  // memory (the common case); if they overflow it but fit the workspace, one
  // more 11-bit digit of the key splits them first: the digits above the
  // threshold digit go straight out and only the threshold digit's candidates
  // are kept in shared memory; otherwise (very many equal keys) the row is
  // rescanned for every level.
  bool in_smem = n_cand <= (uint32_t)kTopkCap;
  uint32_t n_sm = in_smem ? n_cand : 0, need = need0;
  uint64_t pre0 = 0;
  int dec0 = 0;
  int32_t* __restrict__ dst = mid + above;
  if (in_smem) {
    for (uint32_t i = tid; i < n_cand; i += kHistThreads) scand[i] = __ldcg(&cand[i]);
  } else if (n_cand <= cand_cap) {
    constexpr int kU = 4;
    for (int i = tid; i < kBins; i += kHistThreads) h[i] = 0;
    if (tid == 0) {
      s_base_u = 0;
      s_base_e = 0;
    }
    __syncthreads();
    for (uint32_t b = warp * 32 * kU; b < n_cand; b += kHistThreads * kU) {
      uint64_t c[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) c[u] = b + lane + 32 * u < n_cand ? __ldcg(&cand[b + lane + 32 * u]) : 0;
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (b + lane + 32 * u < n_cand) atomicAdd(&h[(uint32_t)(c[u] >> 42) & (kBins - 1)], 1u);
    }
    __syncthreads();
    int d1;
    uint32_t above1;
    find_threshold<kHistThreads>(h, need0, d1, above1, &s_bin, &s_above, s_warp);
    const uint32_t below = (1u << lane) - 1u;
    for (uint32_t b = warp * 32 * kU; b < n_cand; b += kHistThreads * kU) {
      uint64_t c[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) c[u] = b + lane + 32 * u < n_cand ? __ldcg(&cand[b + lane + 32 * u]) : 0;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const bool ok = b + lane + 32 * u < n_cand;
        const int dg = (int)((uint32_t)(c[u] >> 42) & (kBins - 1));
        const uint32_t mu = __ballot_sync(0xffffffffu, ok && dg > d1);
        const uint32_t me = __ballot_sync(0xffffffffu, ok && dg == d1);
        uint32_t bu = 0, be = 0;
        if (lane == 0) {
          if (mu) bu = atomicAdd(&s_base_u, __popc(mu));
          if (me) be = atomicAdd(&s_base_e, __popc(me));
        }
        bu = __shfl_sync(0xffffffffu, bu, 0) + __popc(mu & below);
        be = __shfl_sync(0xffffffffu, be, 0) + __popc(me & below);
        if (ok && dg > d1) {
          if (bu < above1) dst[bu] = (int32_t)(0xFFFFFFFFu - (uint32_t)c[u]);
        } else if (ok && dg == d1) {
          if (be < (uint32_t)kTopkCap) scand[be] = c[u];
        }
      }
    }
    __syncthreads();
    const uint32_t n2 = s_base_e;
    if (n2 <= (uint32_t)kTopkCap) {
      in_smem = true;
      n_sm = n2;
      pre0 = (uint64_t)d1;
      dec0 = 11;
      need = need0 - above1;
      dst += above1;
    }
  }
  __syncthreads();
  auto for_each = [&](auto&& f) {
    if (in_smem) {
      for (uint32_t i = tid; i < n_sm; i += kHistThreads) {
        const uint64_t c = scand[i];
        f(c & kLow53, (int64_t)(0xFFFFFFFFu - (uint32_t)c));
      }
    } else {  // more equal-key scores than the buffers hold: rescan the row
      for (int64_t j = g.lo + tid; j < g.hi; j += kHistThreads) {
        const uint32_t k2 = score_key(srow[j]);
        if ((int)(k2 >> 21) == bin) f((((uint64_t)k2 << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j)) & kLow53, j);
      }
    }
  };
  uint64_t prefix;
  int decided;
  radix_levels<kHistThreads>(for_each, need, h, &s_bin, &s_above, s_warp, prefix, decided, pre0, dec0);
  const int shb = 53 - decided;
  for_each([&](uint64_t v, int64_t j) {
    if ((v >> shb) >= prefix) {
      const uint32_t slot = atomicAdd(&s_slot, 1u);
      if (slot < need) dst[slot] = (int32_t)j;
    }
  });
  // every CTA of the row has taken its ticket: the counters are free again
  if (tid == 0) {
    ctl[0] = 0;
    *reinterpret_cast<unsigned long long*>(&ctl[4]) = 0ull;
  }
}

// One CTA per row: histogram (unless the indexer already built it), threshold,
// one collect pass, and the rest of the select on candidates kept in shared
// memory. For rows up to a few hundred thousand columns this is one launch
// instead of three; the multi-CTA kernels above serve few, very long rows.
constexpr int kRowThreads = 512;
constexpr int kRowCap = 4608;  // 36 KB of candidates: static shared memory stays under 48 KB
constexpr int64_t kSampledMin = 65536;  // middle columns from which a row takes the sampled bound

// kSampled: the instance for long rows without a histogram (below), launched
// only when some row is long enough to use it; the other instance is compiled
// without that path.
template <bool kSampled>
__global__ void __launch_bounds__(kRowThreads, 2) topk_row_kernel(TopkArgs a, int row0, const uint32_t* hist_in) {
  __shared__ uint32_t h[kBins];
  __shared__ uint64_t cand[kRowCap];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_warp[kRowThreads / 32], s_up, s_nc, s_slot;
  __shared__ uint32_t s_wu[kRowThreads / 32], s_we[kRowThreads / 32];
  extern __shared__ int32_t s_map[];  // the row's column map (col_ld entries) when there is one
  pdl_wait();
  pdl_trigger();  // dependents may launch now; they wait for this grid before reading its outputs
  const int r = row0 + blockIdx.x;
  const RowGeom g = row_geom(a, r);
  int32_t* __restrict__ out = a.idx + (int64_t)r * a.topk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (a.zero_hist)
    for (int i = tid; i < kBins; i += kRowThreads) a.zero_hist[(int64_t)r * kTopkHistStride + i] = 0;
  if (a.col_map) {
    for (int i = tid; i < a.col_ld; i += kRowThreads) s_map[i] = a.col_map[(int64_t)r * a.col_ld + i];
    __syncthreads();
  }
  auto col = [&](int64_t j) -> int32_t {  // (a mapped row is shorter than 2^31: 32-bit division)
    if (!a.col_map) return (int32_t)j;
    const uint32_t ju = (uint32_t)j, cb = (uint32_t)a.col_block, q = ju / cb;
    return s_map[q] * a.col_block + (int32_t)(ju - q * cb);
  };
  if (g.dense) {
    for (int i = tid; i < a.topk; i += kRowThreads) out[i] = (i < g.n) ? col(i) : -1;
    if (tid == 0) a.count[r] = (int32_t)g.n;
    return;
  }
  for (int i = tid; i < a.n_init; i += kRowThreads) out[i] = col(i);
  for (int i = tid; i < a.n_loc; i += kRowThreads) out[a.n_init + i] = col(g.hi + i);
  if (tid == 0) {
    a.count[r] = a.topk;
    s_up = 0;
    s_nc = 0;
    s_slot = 0;
  }
  const float* __restrict__ srow = a.scores + (int64_t)r * a.ld;
  const uint32_t k_rem = (uint32_t)(a.topk - a.n_init - a.n_loc);
  // Short rows (at most 16 middle scores per thread): every score is requested
  // at once, before the histogram and the threshold search, and the collect
  // places each thread's scores with one block-wide prefix sum.
  constexpr int kShort = 2 * kUnroll;
  static_assert((int64_t)kRowThreads * kShort == kTopkShortMid, "short rows as the launcher sees them");
  const bool short_row = g.hi - g.lo <= (int64_t)kRowThreads * kShort;
  auto scol = [&](int i) -> int64_t {  // warp w, round q: columns lo + 4096 q + 256 w .. + 255
    return g.lo + (int64_t)(i / kUnroll) * kRowThreads * kUnroll + warp * 32 * kUnroll + lane + 32 * (i % kUnroll);
  };
  float sv[kShort];
  if (short_row) {
#pragma unroll
    for (int i = 0; i < kShort; ++i) {
      const int64_t j = scol(i);
      sv[i] = j < g.hi ? srow[j] : 0.f;
    }
  }
  // Streams the middle columns [lo, hi) in rounds of 8 values per lane:
  // fn(v, jc) with jc(i) the column of v[i] (valid when lo <= jc(i) < hi). When
  // the row is long and 16-byte aligned a warp loads 512 consecutive scores per step
  // (four 16-byte loads per lane in flight, two rounds), else 256 (eight 4-byte
  // loads per lane, one round). The 16-byte loads start at lo rounded down to 4
  // and end at hi rounded up to 4, inside the row since ld is a multiple of 4.
  const bool vec = g.hi - g.lo >= 32768 && (a.ld & 3) == 0 && (reinterpret_cast<uintptr_t>(srow) & 15u) == 0;
  const int64_t hi4 = (g.hi + 3) & ~int64_t(3);  // a load at j4 (a multiple of 4) is below hi iff j4 < hi4
  auto stream_row = [&](auto&& fn) {
    if (vec) {
      for (int64_t base = (g.lo & ~int64_t(3)) + (int64_t)warp * 512; base < g.hi;
           base += (int64_t)kRowThreads * 16) {
        float4 q[4];
        if (kSampled && base + 512 <= hi4) {  // every load of the step below hi: no per-load test
#pragma unroll
          for (int u = 0; u < 4; ++u) q[u] = *reinterpret_cast<const float4*>(srow + base + 128 * u + 4 * lane);
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int64_t j4 = base + 128 * u + 4 * lane;
            q[u] = j4 < g.hi ? *reinterpret_cast<const float4*>(srow + j4) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float v[8] = {q[2 * hf].x,     q[2 * hf].y,     q[2 * hf].z,     q[2 * hf].w,
                              q[2 * hf + 1].x, q[2 * hf + 1].y, q[2 * hf + 1].z, q[2 * hf + 1].w};
          const int64_t j0 = base + 256 * hf + 4 * lane;
          fn(v, [&](int i) -> int64_t { return j0 + 128 * (i >> 2) + (i & 3); });
        }
      }
    } else {
      for (int64_t base = g.lo + warp * 32 * kUnroll; base < g.hi; base += kRowThreads * kUnroll) {
        float v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int64_t j = base + lane + 32 * u;
          v[u] = j < g.hi ? srow[j] : 0.f;
        }
        fn(v, [&](int i) -> int64_t { return base + lane + 32 * i; });
      }
    }
  };
  auto valid = [&](int64_t j) { return j >= g.lo && j < g.hi; };
  const uint32_t below = (1u << lane) - 1u;
  const uint32_t* hr = hist_in ? hist_in + (int64_t)r * kTopkHistStride : nullptr;

  // Long rows without a histogram: a sample sets a bound, one pass collects every
  // score above it, and the selection finishes on those candidates in shared
  // memory. The sample is 64 runs of 256 consecutive middle columns spread over
  // the row; its histogram of the top 13 key bits (a sixteenth of an octave a
  // bin) gives the bound that about twice the budget's share of the sample
  // passes. If at least the budget and at most kRowCap scores pass it, the
  // selection is exact among them (the budget's best all pass); otherwise the
  // two-pass path below runs as if nothing had happened. One pass over the row
  // (plus the sample) instead of two.
  if constexpr (kSampled) if (!hr && !short_row && !a.col_map && g.hi - g.lo >= kSampledMin) {
    __syncthreads();  // s_up / s_nc / s_slot initialised
    constexpr int kSegs = 64, kSegLen = 256, kSBins = 8192;
    uint32_t* hs = reinterpret_cast<uint32_t*>(cand);  // the candidate buffer, free until the collect
    for (int i = tid; i < kSBins; i += kRowThreads) hs[i] = 0;
    __syncthreads();
    const int64_t span = g.hi - g.lo - kSegLen;
    for (int sg = warp; sg < kSegs; sg += kRowThreads / 32) {
      const int64_t s0 = g.lo + span * sg / (kSegs - 1);
      float v[kSegLen / 32];
#pragma unroll
      for (int u = 0; u < kSegLen / 32; ++u) v[u] = srow[s0 + lane + 32 * u];
#pragma unroll
      for (int u = 0; u < kSegLen / 32; ++u) atomicAdd(&hs[score_key(v[u]) >> 19], 1u);
    }
    __syncthreads();
    const uint32_t target =
        (uint32_t)(2.0 * k_rem * (double)(kSegs * kSegLen) / (double)(g.hi - g.lo)) + 16u;
    int b13;
    uint32_t a13;
    find_threshold<kRowThreads, kSBins>(hs, target, b13, a13, &s_bin, &s_above, s_warp);
    // every middle score at or above the bound into shared memory. The bound as
    // a float: the lowest value whose key has top 13 bits b13 (score_key is
    // monotonic), so most rounds cost one compare per score and one vote; the
    // forced columns the 16-byte loads also cover (+inf) only reach the exact
    // test below.
    const uint32_t kmin = (uint32_t)b13 << 19;
    const float tb = __uint_as_float((kmin & 0x80000000u) ? (kmin & 0x7FFFFFFFu) : ~kmin);
    // About twice the budget's share of the scores passes, so a 256-score
    // round holds a passing score more often than not: each of the 8 values
    // then takes its own vote, and only a value with a passing lane pays for
    // the key, the range test and the append.
    stream_row([&](const float(&v)[8], auto jc) {
      float mx = v[0];
#pragma unroll
      for (int u = 1; u < 8; ++u) mx = fmaxf(mx, v[u]);
      if (!__any_sync(0xffffffffu, mx >= tb)) return;  // rounds without a passing score: one vote
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (!__any_sync(0xffffffffu, v[u] >= tb)) continue;
        const uint32_t key = score_key(v[u]);
        const bool take = v[u] >= tb && valid(jc(u)) && (int)(key >> 19) >= b13;
        const uint32_t m = __ballot_sync(0xffffffffu, take);
        if (m == 0) continue;
        uint32_t b = 0;
        if (lane == 0) b = atomicAdd(&s_nc, (uint32_t)__popc(m));
        b = __shfl_sync(0xffffffffu, b, 0) + __popc(m & below);
        if (take && b < (uint32_t)kRowCap) cand[b] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)jc(u));
      }
    });
    __syncthreads();
    const uint32_t n_c = s_nc;
    if (n_c >= k_rem && n_c <= (uint32_t)kRowCap) {
      // the candidates' top 11 bits: the threshold bin among them
      for (int i = tid; i < kBins; i += kRowThreads) h[i] = 0;
      __syncthreads();
      for (uint32_t i = tid; i < n_c; i += kRowThreads) atomicAdd(&h[(uint32_t)(cand[i] >> 53)], 1u);
      __syncthreads();
      int bt;
      uint32_t at;
      find_threshold<kRowThreads>(h, k_rem, bt, at, &s_bin, &s_above, s_warp);
      int32_t* __restrict__ mid = out + a.n_init + a.n_loc;
      for (uint32_t i = tid; i < n_c; i += kRowThreads) {
        const uint64_t c = cand[i];
        if ((int)(c >> 53) > bt) {
          const uint32_t slot = atomicAdd(&s_up, 1u);
          if (slot < at) mid[slot] = (int32_t)(0xFFFFFFFFu - (uint32_t)c);
        }
      }
      auto for_bin = [&](auto&& f) {
        for (uint32_t i = tid; i < n_c; i += kRowThreads) {
          const uint64_t c = cand[i];
          if ((int)(c >> 53) == bt) f(c & kLow53, (int64_t)(0xFFFFFFFFu - (uint32_t)c));
        }
      };
      uint64_t prefix;
      int decided;
      const uint32_t need = k_rem - at;
      radix_levels<kRowThreads>(for_bin, need, h, &s_bin, &s_above, s_warp, prefix, decided);
      const int shb = 53 - decided;
      int32_t* __restrict__ dst = mid + at;
      for_bin([&](uint64_t v, int64_t j) {
        if ((v >> shb) >= prefix) {
          const uint32_t slot = atomicAdd(&s_slot, 1u);
          if (slot < need) dst[slot] = (int32_t)j;
        }
      });
      return;
    }
    __syncthreads();
    if (tid == 0) s_nc = 0;  // the bound missed: the exact two-pass path
  }

  int bin0 = 0;
  uint32_t above0 = 0;
  if (hr) {
    for (int i = tid; i < kBins; i += kRowThreads) h[i] = hr[i];
    __syncthreads();
  } else {
    for (int i = tid; i < kBins; i += kRowThreads) h[i] = 0;
    __syncthreads();
    if (short_row) {
#pragma unroll
      for (int i = 0; i < kShort; ++i)
        if (scol(i) < g.hi) atomicAdd(&h[score_key(sv[i]) >> 21], 1u);
    } else {
      stream_row([&](const float(&v)[8], auto jc) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (valid(jc(u))) atomicAdd(&h[score_key(v[u]) >> 21], 1u);
      });
    }
    __syncthreads();
  }
  find_threshold<kRowThreads>(h, k_rem, bin0, above0, &s_bin, &s_above, s_warp);
  __syncthreads();  // s_up / s_nc initialised
  int32_t* __restrict__ mid = out + a.n_init + a.n_loc;

  if (short_row) {
    // collect of a short row: each thread's counts above and in the threshold
    // bin, exclusive prefix sums over the block, then every score to its place
    uint32_t nu = 0, ne = 0;
#pragma unroll
    for (int i = 0; i < kShort; ++i) {
      const int kb = scol(i) < g.hi ? (int)(score_key(sv[i]) >> 21) : -1;
      nu += kb > bin0;
      ne += kb == bin0;
    }
    uint32_t iu = nu, ie = ne;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t yu = __shfl_up_sync(0xffffffffu, iu, off), ye = __shfl_up_sync(0xffffffffu, ie, off);
      if (lane >= off) {
        iu += yu;
        ie += ye;
      }
    }
    if (lane == 31) {
      s_wu[warp] = iu;
      s_we[warp] = ie;
    }
    __syncthreads();
    uint32_t ou = iu - nu, oe = ie - ne;
    for (int w2 = 0; w2 < warp; ++w2) {
      ou += s_wu[w2];
      oe += s_we[w2];
    }
    if (tid == kRowThreads - 1) s_nc = oe + ne;  // the last thread's prefix is the total
    // branch-free (predicated stores): one straight run of code for all 16
#pragma unroll
    for (int i = 0; i < kShort; ++i) {
      const int64_t j = scol(i);
      const uint32_t key = score_key(sv[i]);
      const int kb = j < g.hi ? (int)(key >> 21) : -1;
      const bool up = kb > bin0, eq = kb == bin0;
      if (up && ou < k_rem) mid[ou] = col(j);
      if (eq && oe < (uint32_t)kRowCap) cand[oe] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
      ou += up;
      oe += eq;
    }
  } else {
  // collect: higher bins straight out, the threshold bin into shared memory
  // (one pair of shared atomics per warp and round: the round's counts first).
  // Only a few thousand of a row's scores reach the threshold bin: a round in
  // which no lane of the warp has one costs one vote.
  const uint32_t kmin0 = (uint32_t)bin0 << 21;  // the threshold bin's lowest value as a float (see above)
  const float tb0 = __uint_as_float((kmin0 & 0x80000000u) ? (kmin0 & 0x7FFFFFFFu) : ~kmin0);
  stream_row([&](const float(&v)[8], auto jc) {
    uint32_t key[8], upm[8], eqm[8];
    bool hit = false;
#pragma unroll
    for (int u = 0; u < 8; ++u) hit |= v[u] >= tb0;
    if (!__any_sync(0xffffffffu, hit)) return;
#pragma unroll
    for (int u = 0; u < 8; ++u) key[u] = score_key(v[u]);
    uint32_t n_up = 0, n_eq = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const bool ok = valid(jc(u));
      const int kb = ok ? (int)(key[u] >> 21) : -1;
      upm[u] = __ballot_sync(0xffffffffu, kb > bin0);
      eqm[u] = __ballot_sync(0xffffffffu, kb == bin0);
      n_up += __popc(upm[u]);
      n_eq += __popc(eqm[u]);
    }
    uint32_t b_up = 0, b_eq = 0;
    if (lane == 0) {
      if (n_up) b_up = atomicAdd(&s_up, n_up);
      if (n_eq) b_eq = atomicAdd(&s_nc, n_eq);
    }
    b_up = __shfl_sync(0xffffffffu, b_up, 0);
    b_eq = __shfl_sync(0xffffffffu, b_eq, 0);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int64_t j = jc(u);
      if ((upm[u] >> lane) & 1u) {
        const uint32_t slot = b_up + __popc(upm[u] & below);
        if (slot < k_rem) mid[slot] = col(j);
      } else if ((eqm[u] >> lane) & 1u) {
        const uint32_t slot = b_eq + __popc(eqm[u] & below);
        if (slot < (uint32_t)kRowCap) cand[slot] = ((uint64_t)key[u] << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
      }
      b_up += __popc(upm[u]);
      b_eq += __popc(eqm[u]);
    }
  });
  }
  __syncthreads();
  const uint32_t need0 = k_rem - above0;
  uint32_t n_cand = s_nc, need = need0;
  bool in_smem = n_cand <= (uint32_t)kRowCap;
  uint64_t pre0 = 0;
  int dec0 = 0;
  int32_t* __restrict__ dst = mid + above0;
  if (!in_smem) {
    // The threshold bin outgrew shared memory: one more 11-bit digit of the
    // key (key bits 20..10) splits it. A histogram pass and a collect pass over
    // the row send the digits above the threshold digit straight out and keep
    // the threshold digit's candidates in shared memory.
    for (int i = tid; i < kBins; i += kRowThreads) h[i] = 0;
    __syncthreads();
    stream_row([&](const float(&v)[8], auto jc) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t key = score_key(v[u]);
        if (valid(jc(u)) && (int)(key >> 21) == bin0) atomicAdd(&h[(key >> 10) & (kBins - 1)], 1u);
      }
    });
    __syncthreads();
    int d1;
    uint32_t above1;
    find_threshold<kRowThreads>(h, need0, d1, above1, &s_bin, &s_above, s_warp);
    if (tid == 0) {
      s_up = 0;
      s_nc = 0;
    }
    __syncthreads();
    stream_row([&](const float(&v)[8], auto jc) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t j = jc(u);
        const uint32_t key = score_key(v[u]);
        const bool inb = valid(j) && (int)(key >> 21) == bin0;
        const int dg = (int)((key >> 10) & (kBins - 1));
        const uint32_t mu = __ballot_sync(0xffffffffu, inb && dg > d1);
        const uint32_t me = __ballot_sync(0xffffffffu, inb && dg == d1);
        uint32_t bu = 0, be = 0;
        if (lane == 0) {
          if (mu) bu = atomicAdd(&s_up, __popc(mu));
          if (me) be = atomicAdd(&s_nc, __popc(me));
        }
        bu = __shfl_sync(0xffffffffu, bu, 0) + __popc(mu & below);
        be = __shfl_sync(0xffffffffu, be, 0) + __popc(me & below);
        if (inb && dg > d1) {
          if (bu < above1) dst[bu] = col(j);
        } else if (inb && dg == d1) {
          if (be < (uint32_t)kRowCap) cand[be] = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
        }
      }
    });
    __syncthreads();
    if (s_nc <= (uint32_t)kRowCap) {
      in_smem = true;
      n_cand = s_nc;
      pre0 = (uint64_t)d1;
      dec0 = 11;
      need = need0 - above1;
      dst += above1;
    }
  }

  auto for_each = [&](auto&& f) {
    if (in_smem) {
      for (uint32_t i = tid; i < n_cand; i += kRowThreads) {
        const uint64_t c = cand[i];
        f(c & kLow53, (int64_t)(0xFFFFFFFFu - (uint32_t)c));
      }
    } else {  // very many equal keys: rescan the row for every level
      for (int64_t j = g.lo + tid; j < g.hi; j += kRowThreads) {
        const uint32_t key = score_key(srow[j]);
        if ((int)(key >> 21) == bin0) {
          const uint64_t c = ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)j);
          f(c & kLow53, j);
        }
      }
    }
  };
  uint64_t prefix;
  int decided;
  radix_levels<kRowThreads>(for_each, need, h, &s_bin, &s_above, s_warp, prefix, decided, pre0, dec0);
  const int sh = 53 - decided;
  for_each([&](uint64_t v, int64_t j) {
    if ((v >> sh) >= prefix) {
      const uint32_t slot = atomicAdd(&s_slot, 1u);
      if (slot < need) dst[slot] = col(j);
    }
  });
}

// Clears n words on the stream as a kernel (a memset between two kernels would
// keep the second from launching while the first finishes).
__global__ void zero_words_kernel(uint32_t* __restrict__ p, size_t n) {
  pdl_wait();  // the previous kernel may still read these words
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0;
  pdl_trigger();
}

}  // namespace

cudaError_t launch_zero_words(void* p, size_t n_words, cudaStream_t st) {
  if (n_words == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)min64(148 * 4, (int64_t)((n_words + 255) / 256));
  count_launches(1);
  return launch_pdl(zero_words_kernel, dim3(blocks), dim3(256), 0, st, static_cast<uint32_t*>(p), n_words);
}

// Dynamic shared memory of the per-row kernel: the column map, if any (at most
// 2048 entries; the attribute allowing it above the 48 KB default is set once).
static size_t row_map_smem(const TopkArgs& a) {
  if (!a.col_map) return 0;
  static bool attr_set = false;  // benign race: every caller sets the same value
  if (!attr_set) {
    cudaFuncSetAttribute(topk_row_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, 2048 * 4);
    attr_set = true;
  }
  return (size_t)a.col_ld * sizeof(int32_t);
}

cudaError_t launch_topk_dense(const TopkArgs& a, cudaStream_t st) {
  // every row is dense: the per-row kernel writes 0..n-1 and the count
  for (int row0 = 0; row0 < a.n_rows; row0 += 65535) {
    const int nr = min(65535, a.n_rows - row0);
    const cudaError_t e = launch_pdl(topk_row_kernel<false>, dim3(nr), dim3(kRowThreads), row_map_smem(a), st, a,
                                     row0, (const uint32_t*)nullptr);
    if (e != cudaSuccess) return e;
    count_launches(1);
  }
  return cudaSuccess;
}

// One CTA per row when there are enough rows to fill the GPU or the rows are
// short; otherwise several CTAs per row. Only the multi-CTA kernels use the
// workspace.
bool topk_uses_workspace(int n_rows, int64_t max_len) { return n_rows < 256 && max_len > (int64_t)16384; }

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t st) {
  if (a.n_rows <= 0) return cudaSuccess;
  if (a.max_len <= a.topk) return launch_topk_dense(a, st);
  const int64_t chunks = (a.max_len + kChunk - 1) / kChunk;
  HistCtl* hc = static_cast<HistCtl*>(a.ws);
  const bool per_row = !topk_uses_workspace(a.n_rows, a.max_len) || a.col_map != nullptr || a.zero_hist != nullptr;
  if (per_row) {
    const uint32_t* hist_in = a.hist_ext;
    // some row may take the sampled bound: no histogram given, long enough, no column map
    const bool sampled = !hist_in && !a.col_map && a.max_len - a.n_init - a.n_loc >= kSampledMin;
    for (int row0 = 0; row0 < a.n_rows; row0 += 65535) {
      const int nr = min(65535, a.n_rows - row0);
      const cudaError_t e =
          sampled ? launch_pdl(topk_row_kernel<true>, dim3(nr), dim3(kRowThreads), 0, st, a, row0, hist_in)
                  : launch_pdl(topk_row_kernel<false>, dim3(nr), dim3(kRowThreads), row_map_smem(a), st, a, row0,
                               hist_in);
      if (e != cudaSuccess) return e;
      count_launches(1);
    }
    return cudaGetLastError();
  }
  const int64_t rows_fit = (int64_t)(a.ws_bytes / kTopkRowBytes);
  const int blk = (int)min64(min64(rows_fit, a.n_rows), 65535);
  uint64_t* cand = reinterpret_cast<uint64_t*>(hc + blk);
  // candidates per row: all the workspace holds beyond the control blocks (at least kTopkCap)
  const uint32_t cand_cap =
      (uint32_t)min64((int64_t)((a.ws_bytes - (size_t)blk * sizeof(HistCtl)) / ((size_t)blk * sizeof(uint64_t))),
                      int64_t(1) << 24);
  for (int row0 = 0; row0 < a.n_rows; row0 += blk) {
    const int nr = min(blk, a.n_rows - row0);
    cudaError_t e = cudaSuccess;
    if (!a.hist_ext) {  // (with the indexer's histograms the counters live beside them)
      e = launch_zero_words(hc, (size_t)nr * sizeof(HistCtl) / sizeof(uint32_t), st);
      if (e != cudaSuccess) return e;
      e = launch_pdl(topk_hist_kernel, dim3((unsigned)chunks, (unsigned)nr), dim3(kHistThreads), 0, st, a, row0, hc);
      if (e != cudaSuccess) return e;
      count_launches(1);
    }
    e = launch_pdl(topk_select_kernel, dim3((unsigned)chunks, (unsigned)nr), dim3(kHistThreads), 0, st, a, row0, hc,
                   cand, cand_cap);
    if (e != cudaSuccess) return e;
    count_launches(1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_topk_hist_only(const TopkArgs& a, uint32_t* hist, cudaStream_t st) {
  if (a.n_rows <= 0 || a.max_len <= a.topk) return cudaSuccess;
  static_assert(sizeof(HistCtl) == kTopkHistStride * sizeof(uint32_t), "histogram row stride");
  const int64_t chunks = (a.max_len + kChunk - 1) / kChunk;
  HistCtl* hc = reinterpret_cast<HistCtl*>(hist);
  for (int row0 = 0; row0 < a.n_rows; row0 += 65535) {
    const int nr = min(65535, a.n_rows - row0);
    const cudaError_t e = launch_pdl(topk_hist_kernel, dim3((unsigned)chunks, (unsigned)nr), dim3(kHistThreads), 0,
                                     st, a, row0, hc + row0);
    if (e != cudaSuccess) return e;
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace lsa
