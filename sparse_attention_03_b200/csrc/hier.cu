// Hierarchical indexing: block summaries and the glue of the two-stage selection.
//
// [LSA-2.0] "分层索引": coarse-to-fine two-stage scoring, approximate
// block-level scores first, then token-level selection inside the surviving
// blocks, which shrinks the candidate space the indexer handles.
// Readings (the page gives the structure only): a block is `block` consecutive
// cached keys of one sequence; its summary key is the mean of its keys,
// rounded once to bf16; the coarse stage is the flat selection one level up
// (sink and most recent blocks forced, the n_blocks best others kept); the
// fine stage is the flat selection over the kept blocks' tokens.
//
// The coarse scores come from the streaming indexer run over the summaries
// (row positions divided by the block size as it reads them), the coarse and
// fine selections from the flat top-k (the fine one mapping compact slots back
// to token columns as it writes them); this file holds the summaries.
#include "common.cuh"
#include "index_tile.cuh"
#include "kernels.h"
#include "launch.h"

namespace lsa {
namespace {

// fp64 -> bf16 bits, round to nearest even, from the IEEE binary64 layout
// (finite inputs in bf16's normal range; bf16 keeps 7 of the 52 fraction bits).
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const uint64_t b = (uint64_t)__double_as_longlong(x);
  const uint64_t sign = b >> 63;
  const int exp = (int)((b >> 52) & 0x7ff);
  if (exp == 0) return (uint16_t)(sign << 15);  // zero (and fp64 subnormals, far below bf16's range)
  const uint64_t drop = 52 - 7;
  const uint64_t mag = b & 0x7fffffffffffffffull;
  const uint64_t r = (mag + (1ull << (drop - 1)) - 1 + ((mag >> drop) & 1)) >> drop;  // rounded, exponent included
  // r = (fp64 exponent << 7) | 7 fraction bits; rebias 1023 -> 127
  const int64_t e = (int64_t)(r >> 7) - 1023 + 127;
  const uint32_t frac = (uint32_t)(r & 0x7f);
  uint32_t out;
  if (e >= 0xff) out = 0x7f80;              // overflow -> inf
  else if (e <= 0) out = 0;                 // below bf16's normal range -> zero
  else out = ((uint32_t)e << 7) | frac;
  return (uint16_t)((sign << 15) | out);
}

// One CTA per item: the mean of the block's keys. Thread (grp, c) sums keys
// grp, grp + 16, ... over dims 8c .. 8c + 7 with 16-byte loads (every load of the
// block in flight at once), then the 16 partial sums of each dim are added in a
// fixed order (the fp64 sums are exact, so the order does not change them).
constexpr int kSumThreads = 256;
constexpr int kSumGroups = kSumThreads / (kDi / 8);  // 16 key groups

__global__ void __launch_bounds__(kSumThreads) block_summary_kernel(BlockSumArgs a) {
  __shared__ double part[kSumGroups][kDi];
  pdl_wait();
  const int i = blockIdx.x, tid = threadIdx.x;
  const int grp = tid / (kDi / 8), c = tid % (kDi / 8);
  const int s = a.item_seq[i];
  if (s < 0 || s >= a.n_seq) {
    if (tid == 0) flag_error(a.err, LSA_DEVERR_SEQ);
    return;
  }
  const int64_t base = a.k_off[s], len = a.k_off[s + 1] - base;
  const int64_t bbase = a.blk_off[s], nb = a.blk_off[s + 1] - bbase;
  const int64_t b = a.item_blk[i];
  const int64_t t0 = b * a.block, t1 = min64(t0 + a.block, len);
  if (b < 0 || b >= nb || t0 >= len) {
    if (tid == 0) flag_error(a.err, LSA_DEVERR_POS);
    return;
  }
  const int n = (int)(t1 - t0);
  const uint4* __restrict__ k = reinterpret_cast<const uint4*>(a.k_idx + (base + t0) * kDi) + c;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int t = grp; t < n; t += kSumGroups * 4) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = t + u * kSumGroups < n ? __ldg(k + (int64_t)(t + u * kSumGroups) * (kDi / 8))
                                                              : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += (double)__uint_as_float(w[e] << 16);
        acc[2 * e + 1] += (double)__uint_as_float(w[e] & 0xffff0000u);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[grp][8 * c + e] = acc[e];
  __syncthreads();
  if (tid < kDi) {
    double sum = 0.0;
#pragma unroll
    for (int g2 = 0; g2 < kSumGroups; ++g2) sum += part[g2][tid];
    a.k_blk[(bbase + b) * kDi + tid] = f64_to_bf16_rne(sum / (double)n);
  }
  pdl_trigger();
}

using namespace idx;
constexpr int kMaxHierBlocks = 2048;  // kept blocks per row (the top-k's own limit)

// ---------------------------------------------------------------------------
// Hierarchical indexing, fine stage ([LSA-2.0] "分层索引"): the same scoring
// over only the tokens of each row's kept blocks, written to a compact row
// (slot i = token sorted[i / block] * block + i % block, blocks in ascending
// order so that the top-k's lower-slot tie rule is the lower-column rule).
// The kept blocks always include the sink blocks (first in order) and the most
// recent blocks (last, consecutive), so in compact slots the sink tokens are
// 0 .. init-1 and the local window is the `local` slots ending at the slot of
// the row's own token, pos_c: the flat top-k then applies its own forcing to
// the compact row with position pos_c, and only the tokens in between are
// scored here. Each CTA also adds those slots to the compact row's top-k
// histogram (the top 11 bits of each score key, as the top-k's first pass
// would count its middle columns).
__global__ void __launch_bounds__(kThreads, 3) hier_fine_kernel(HierFineArgs h, int blocks_per_cta) {
  __shared__ int32_t ids[kMaxHierBlocks];
  __shared__ int32_t srt[kMaxHierBlocks];
  __shared__ uint32_t sh[2048];   // the kept blocks as a bitmap, then the histogram
  __shared__ uint32_t pre[2048];  // set bits in the bitmap's earlier words
  pdl_wait();
  const IndexArgs& a = h.ix;
  const int r = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;

  // row geometry, clamped and flagged as in the flat indexer; the query
  // fragments and head weights are requested before the kept list is sorted
  const int seq = a.seq_of_row ? a.seq_of_row[r] : (a.seq_identity ? r : 0);
  int64_t kbase = 0, klen = a.max_len;
  bool ok = true;
  if (seq < 0 || seq >= a.n_seq) {
    ok = false;
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(a.err, LSA_DEVERR_SEQ);
  } else if (a.k_off) {
    kbase = a.k_off[seq];
    klen = a.k_off[seq + 1] - kbase;
  }
  const int64_t p = a.pos[r];
  int64_t nvis = p + 1;
  if (ok && (p < 0 || nvis > klen || nvis > a.max_len)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(a.err, LSA_DEVERR_POS);
    nvis = max64(0, min(nvis, min(klen, a.max_len)));
  }
  if (!ok) nvis = 0;
  uint4 qf[4][4];
  const uint16_t* __restrict__ qr = a.q_idx + (int64_t)r * kHi * kDi;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c)
      qf[nt][c] = __ldg(reinterpret_cast<const uint4*>(qr + (8 * nt + g) * kDi + 8 * (4 * c + t)));
  float wf[4][2];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) wf[nt][e] = __ldg(a.w + (int64_t)r * kHi + 8 * nt + 2 * t + e);

  // the kept blocks in ascending order (the ids of a row are distinct; clamping
  // and pre-filling keep every token index in range even for a malformed list):
  // ranks from a bitmap of the ids and its prefix counts when the ids fit in
  // 65536 bits, else by counting
  const int n = min(h.kept_n[r], h.kb);
  const int32_t* __restrict__ kr = h.kept + (int64_t)r * h.kb;
  const bool bitmap = h.nb_max <= 2048 * 32;
  const int n_words = bitmap ? (int)((h.nb_max + 31) / 32) : 0;
  for (int i = threadIdx.x; i < n; i += kThreads) {
    ids[i] = min(max(kr[i], 0), (int)max64(h.nb_max - 1, 0));
    srt[i] = 0;
  }
  for (int i = threadIdx.x; i < n_words; i += kThreads) sh[i] = 0;
  __syncthreads();
  if (bitmap) {
    for (int i = threadIdx.x; i < n; i += kThreads) atomicOr(&sh[ids[i] >> 5], 1u << (ids[i] & 31));
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of the words' popcounts, 32 words per step
      uint32_t carry = 0;
      for (int w0 = 0; w0 < n_words; w0 += 32) {
        const uint32_t c = w0 + lane < n_words ? (uint32_t)__popc(sh[w0 + lane]) : 0u;
        uint32_t x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (w0 + lane < n_words) pre[w0 + lane] = carry + x - c;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const int v = ids[i];
      srt[pre[v >> 5] + __popc(sh[v >> 5] & ((1u << (v & 31)) - 1u))] = v;
    }
  } else {
    for (int i = threadIdx.x; i < n; i += kThreads) {
      const int v = ids[i];
      int rank = 0;
      for (int j = 0; j < n; ++j) rank += ids[j] < v;
      srt[rank] = v;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2048; i += kThreads) sh[i] = 0;  // now the histogram
  __syncthreads();
  const bool dense_row = p >= 0 && p + 1 <= h.topk;
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < n; i += kThreads) h.sorted[(int64_t)r * h.kb + i] = srt[i];
    // the row's own token is in the last kept block (a dense row keeps every
    // block, so there pos_c = pos); -1 for a row with no visible key
    if (threadIdx.x == 0) h.pos_c[r] = (n > 0 && nvis > 0) ? (n - 1) * h.block + (int32_t)((nvis - 1) % h.block) : -1;
  }

  const int64_t s_lo = (int64_t)blockIdx.x * blocks_per_cta * h.block;
  const int64_t s_hi = min((int64_t)(blockIdx.x + 1) * blocks_per_cta, (int64_t)n) * h.block;
  const uint16_t* __restrict__ kb = a.k_idx + kbase * kDi;
  const int64_t lo_force = a.n_init, hi_force = p + 1 - a.n_loc;
  float* __restrict__ crow = h.cand + (int64_t)r * h.ld_c;
  // slot tiles of 16 (a block is a multiple of 16 keys, so a tile never straddles
  // two); a compact row is shorter than 2^31 slots: 32-bit division
  const uint32_t ub = (uint32_t)h.block;
  auto tok = [&](int64_t s) {
    const uint32_t su = (uint32_t)s, q = su / ub;
    return (int64_t)srt[q] * h.block + (int64_t)(su - q * ub);
  };
  // a tile whose tokens are all forced or all past the row's position needs no keys
  auto needs_keys = [&](int64_t s) {
    const int64_t j0 = tok(s);
    return !(j0 + kKeysPerWarpTile <= lo_force || (j0 >= hi_force) || j0 >= nvis);
  };
  auto put = [&](int64_t s, float sa, float sb) {
    if (t < 2) {
      const int64_t j = tok(s) + g + (t == 1 ? 8 : 0);
      const bool forced = (j < lo_force) || (j >= hi_force);
      // forced slots and slots past the row's token are never read by the top-k
      if (j < nvis && !forced) {
        const float v = t == 1 ? sb : sa;
        crow[s + g + (t == 1 ? 8 : 0)] = v;
        atomicAdd(&sh[score_key(v) >> 21], 1u);
      }
    }
  };
  const int64_t step = kWarps * kKeysPerWarpTile;
  int64_t s = s_lo + warp * kKeysPerWarpTile;
  if (s < s_hi) {
    KeyFrag f0, f1;
    const int64_t tend = 0;  // (no key is read for a tile that needs none)
    load_keys(f0, kb, tok(s) + g, needs_keys(s) ? nvis : tend, t);
    while (true) {
      int64_t nxt = s + step;
      if (nxt < s_hi) load_keys(f1, kb, tok(nxt) + g, needs_keys(nxt) ? nvis : tend, t);
      float sa, sb;
      score_tile(f0, qf, wf, sa, sb);
      put(s, sa, sb);
      if (nxt >= s_hi) break;
      s = nxt;
      nxt = s + step;
      if (nxt < s_hi) load_keys(f0, kb, tok(nxt) + g, needs_keys(nxt) ? nvis : tend, t);
      score_tile(f1, qf, wf, sa, sb);
      put(s, sa, sb);
      if (nxt >= s_hi) break;
      s = nxt;
    }
  }
  pdl_trigger();
  __syncthreads();
  if (!dense_row && s_lo < s_hi) {
    uint32_t* __restrict__ hr = h.hist + (int64_t)r * kTopkHistStride;
    for (int i = threadIdx.x; i < 2048; i += kThreads)
      if (sh[i]) atomicAdd(&hr[i], sh[i]);
  }
}


}  // namespace

cudaError_t launch_block_summaries(const BlockSumArgs& a, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  count_launches(1);
  return launch_pdl(block_summary_kernel, dim3(a.n_items), dim3(kSumThreads), 0, st, a);
}

cudaError_t launch_hier_fine(const HierFineArgs& h, cudaStream_t st) {
  if (h.ix.n_rows <= 0) return cudaSuccess;
  if (h.kb > kMaxHierBlocks || h.block % kKeysPerWarpTile != 0) return cudaErrorInvalidValue;
  // one wave of CTAs (three per SM), each a whole number of kept blocks
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t wave = 3LL * sms;
  const int64_t per_row = max64(1, wave / h.ix.n_rows);
  const int bpc = (int)max64(1, (h.kb + per_row - 1) / per_row);
  const int nx = (h.kb + bpc - 1) / bpc;
  for (int row0 = 0; row0 < h.ix.n_rows; row0 += 65535) {
    HierFineArgs b = h;
    const int ny = min(65535, h.ix.n_rows - row0);
    b.ix.n_rows = ny;
    b.ix.pos += row0;
    if (b.ix.seq_of_row) b.ix.seq_of_row += row0;
    b.ix.q_idx += (int64_t)row0 * kHi * kDi;
    b.ix.w += (int64_t)row0 * kHi;
    b.kept += (int64_t)row0 * h.kb;
    b.kept_n += row0;
    b.sorted += (int64_t)row0 * h.kb;
    b.pos_c += row0;
    b.cand += (int64_t)row0 * h.ld_c;
    b.hist += (int64_t)row0 * kTopkHistStride;
    const cudaError_t e = launch_pdl(hier_fine_kernel, dim3(nx, ny), dim3(kThreads), 0, st, b, bpc);
    if (e != cudaSuccess) return e;
    count_launches(1);
  }
  return cudaSuccess;
}

}  // namespace lsa
