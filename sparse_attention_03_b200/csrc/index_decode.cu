// Lightning indexer, streaming form (decode and any row set that does not share keys).
//
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）": per index head q.k, ReLU, then the
// head-weighted sum; sink and local-window columns forced to +inf.
// [Lite-Sparse] "预填充优化": the ReLU-weighted head sum is fused into the
// epilogue so the per-head [heads x keys] tensor is never written.
// [LSA-2.0] "流式感知索引": the key stream is read as contiguous, coalesced HBM
// traffic.
//
// Design. The per-key work is a [32 heads x 128] x [128] contraction (8192 flop
// per 256-byte key row), too much for the FP32 pipes at HBM speed, so the keys
// go through the tensor cores: a warp takes 16 keys as the M dimension of
// mma.m16n8k16 (bf16 in, fp32 accumulate), the 32 heads as four n8 tiles, and
// the 128 dims as eight k16 steps. The query's B fragments stay in registers for
// the whole CTA. Each lane loads its A fragments straight from HBM with 16-byte
// non-allocating loads: the contraction dimension is permuted (identically for
// q and k, which leaves every dot product unchanged) so that one lane's eight
// bf16 pairs of a key row are four contiguous 16-byte chunks, and the four lanes
// of a quad read 64 contiguous bytes per instruction. The ReLU-weighted head sum
// runs on the accumulators in registers, then two quad shuffles finish it.
#include "common.cuh"
#include "kernels.h"
#include "launch.h"

namespace lsa {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kKeysPerWarpTile = 16;
constexpr int kMaxHierBlocks = 2048;  // kept blocks per row (the top-k's own limit)

struct KeyFrag {
  uint4 lo[4];  // key g:   physical dims 8*(4c+t) .. +7, c = 0..3
  uint4 hi[4];  // key g+8
};

__device__ __forceinline__ void load_keys(KeyFrag& f, const uint16_t* __restrict__ kb, int64_t ja,
                                          int64_t jend, int t) {
  const int64_t jb = ja + 8;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    f.lo[c] = (ja < jend) ? ld_stream_v4(kb + ja * kDi + 8 * (4 * c + t)) : make_uint4(0, 0, 0, 0);
    f.hi[c] = (jb < jend) ? ld_stream_v4(kb + jb * kDi + 8 * (4 * c + t)) : make_uint4(0, 0, 0, 0);
  }
}

// Scores of keys g and g+8 of the tile (valid in every lane of the quad).
__device__ __forceinline__ void score_tile(const KeyFrag& f, const uint4 (&qf)[4][4],
                                           const float (&wf)[4][2], float& sa, float& sb) {
  float acc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int c = s >> 1;
    const bool h = (s & 1) != 0;
    // logical k (2t, 2t+1) -> physical elements {0,1} or {4,5} of chunk c;
    // logical k (2t+8, 2t+9) -> physical {2,3} or {6,7}.
    const uint32_t a0 = h ? f.lo[c].z : f.lo[c].x;
    const uint32_t a1 = h ? f.hi[c].z : f.hi[c].x;
    const uint32_t a2 = h ? f.lo[c].w : f.lo[c].y;
    const uint32_t a3 = h ? f.hi[c].w : f.hi[c].y;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const uint32_t b0 = h ? qf[nt][c].z : qf[nt][c].x;
      const uint32_t b1 = h ? qf[nt][c].w : qf[nt][c].y;
      mma_16816(acc[nt], a0, a1, a2, a3, b0, b1);
    }
  }
  // acc[nt][e] = (key g, head 8nt+2t+e); acc[nt][2+e] = (key g+8, same head).
  float x = 0.f, y = 0.f;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      x = fmaf(wf[nt][e], fmaxf(acc[nt][e], 0.f), x);
      y = fmaf(wf[nt][e], fmaxf(acc[nt][2 + e], 0.f), y);
    }
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  y += __shfl_xor_sync(0xffffffffu, y, 1);
  y += __shfl_xor_sync(0xffffffffu, y, 2);
  sa = x;
  sb = y;
}

template <bool HIST>
__global__ void __launch_bounds__(kThreads, 3)
    index_decode_kernel(IndexArgs a, int keys_per_cta, int row0, uint32_t* hist, int topk) {
  __shared__ uint32_t sh[HIST ? 2048 : 1];
  pdl_wait();
  const int r = row0 + blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * keys_per_cta;
  if (j0 >= a.max_len) return;
  const int64_t j1 = min(j0 + (int64_t)keys_per_cta, a.max_len);

  // Row geometry, with every out-of-range input clamped and flagged.
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
  const int pr = a.pos[r];
  const int64_t p = a.pos_div == 1 ? pr : (pr >= 0 ? pr / a.pos_div : -1);
  int64_t nvis = p + 1;
  if (ok && (p < 0 || nvis > klen || nvis > a.max_len)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(a.err, LSA_DEVERR_POS);
    nvis = max64(0, min(nvis, min(klen, a.max_len)));
  }
  if (!ok) nvis = 0;

  float* __restrict__ srow = a.scores + (int64_t)r * a.ld;
  const int64_t jend = min(j1, nvis);  // columns after pos are never written
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  int64_t tile = j0 + warp * kKeysPerWarpTile;
  // The top-k's histogram (top 11 bits of each middle-column score key) of rows
  // that will be selected from, built here from the scores in registers.
  const bool hist_row = HIST && ok && (p + 1 > topk);
  if (HIST) {
    for (int i = threadIdx.x; i < 2048; i += kThreads) sh[i] = 0;
    __syncthreads();
  }
  if (tile < jend) {

  // Query B fragments (head 8nt+g, physical chunk 4c+t) and head weights.
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

  const uint16_t* __restrict__ kb = a.k_idx + kbase * kDi;
  const int64_t step = kWarps * kKeysPerWarpTile;
  const int64_t lo_force = a.n_init, hi_force = p + 1 - a.n_loc;

  auto put = [&](int64_t tl, float sa, float sb) {
    if (t < 2) {
      const int64_t j = tl + g + (t == 1 ? 8 : 0);
      if (j < jend) {
        const bool forced = (j < lo_force) || (j >= hi_force);
        const float v = t == 1 ? sb : sa;
        srow[j] = forced ? INFINITY : v;
        if (HIST && hist_row && !forced) atomicAdd(&sh[score_key(v) >> 21], 1u);
      }
    }
  };

  // Two register sets: the next tile's loads are in flight while this one computes.
  KeyFrag f0, f1;
  load_keys(f0, kb, tile + g, jend, t);
  while (true) {
    int64_t nxt = tile + step;
    if (nxt < jend) load_keys(f1, kb, nxt + g, jend, t);
    float sa, sb;
    score_tile(f0, qf, wf, sa, sb);
    put(tile, sa, sb);
    if (nxt >= jend) break;
    tile = nxt;
    nxt = tile + step;
    if (nxt < jend) load_keys(f0, kb, nxt + g, jend, t);
    score_tile(f1, qf, wf, sa, sb);
    put(tile, sa, sb);
    if (nxt >= jend) break;
    tile = nxt;
  }
  }
  pdl_trigger();
  if (HIST) {
    __syncthreads();
    uint32_t* hr = hist + (int64_t)r * kTopkHistStride;
    for (int i = threadIdx.x; i < 2048; i += kThreads)
      if (sh[i]) atomicAdd(&hr[i], sh[i]);
  }
}


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

cudaError_t launch_index_decode(const IndexArgs& a, cudaStream_t st, uint32_t* hist, int topk) {
  if (a.n_rows <= 0) return cudaSuccess;
  // One wave: as many CTAs as the SMs hold at once (a second, partial wave of
  // these short-lived CTAs costs more than the larger per-CTA key range saves).
  // Keys per CTA are a multiple of one CTA pass (64 keys), at least 256 so the
  // query-fragment load is amortised (64 for rows of at most 16384 keys), and at
  // most 8192.
  // Cached per device (a benign race: every thread writes the same values).
  static int cache_sms[64], cache_occ[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cache_sms[dev] == 0) {
    int s = 148, o = 3;
    cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, index_decode_kernel<true>, kThreads, 0) != cudaSuccess ||
        o < 1)
      o = 3;
    cache_occ[dev] = o;
    cache_sms[dev] = s;
  }
  const int sms = cache_sms[dev], occ = cache_occ[dev];
  const int64_t wave = (int64_t)sms * occ;
  const int64_t per_row = max64(1, wave / a.n_rows);
  int64_t kpc = (a.max_len + per_row - 1) / per_row;
  kpc = ((kpc + 63) / 64) * 64;
  // short rows (block summaries) spread over more CTAs; long ones amortise the
  // query-fragment load over at least 256 keys
  kpc = max64(a.max_len <= 16384 ? 64 : 256, min64(kpc, 8192));
  const int64_t nx = (a.max_len + kpc - 1) / kpc;
  for (int row0 = 0; row0 < a.n_rows; row0 += 65535) {
    const int ny = min(65535, a.n_rows - row0);
    const dim3 grid((unsigned)nx, (unsigned)ny);
    const cudaError_t e =
        hist ? launch_pdl(index_decode_kernel<true>, grid, dim3(kThreads), 0, st, a, (int)kpc, row0, hist, topk)
             : launch_pdl(index_decode_kernel<false>, grid, dim3(kThreads), 0, st, a, (int)kpc, row0,
                          (uint32_t*)nullptr, 0);
    if (e != cudaSuccess) return e;
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace lsa

namespace lsa {

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
