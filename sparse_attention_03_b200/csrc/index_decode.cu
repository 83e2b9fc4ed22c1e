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
// runs on the accumulators in registers, then two quad shuffles finish it. The
// tile code (fragment loads and scoring) is in index_tile.cuh.
#include "common.cuh"
#include "index_tile.cuh"
#include "kernels.h"
#include "launch.h"

namespace lsa {
namespace {

using namespace idx;

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


}  // namespace

cudaError_t launch_index_decode(const IndexArgs& a, cudaStream_t st, uint32_t* hist, int topk) {
  if (a.n_rows <= 0) return cudaSuccess;
  // One wave: as many CTAs as the SMs hold at once (a second, partial wave of
  // these short-lived CTAs costs more than the larger per-CTA key range saves).
  // Keys per CTA are a multiple of one CTA pass (64 keys), at least 256 so the
  // query-fragment load is amortised (64 for rows of at most 16384 keys), and at
  // most 65536 (a few long rows then still fill exactly one wave).
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
  kpc = max64(a.max_len <= 16384 ? 64 : 256, min64(kpc, 65536));
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

