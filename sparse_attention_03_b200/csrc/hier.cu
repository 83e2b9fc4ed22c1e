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

}  // namespace

cudaError_t launch_block_summaries(const BlockSumArgs& a, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  count_launches(1);
  return launch_pdl(block_summary_kernel, dim3(a.n_items), dim3(kSumThreads), 0, st, a);
}

}  // namespace lsa
