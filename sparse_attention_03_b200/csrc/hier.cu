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
// The coarse scores come from the streaming indexer run over the summaries,
// the coarse and fine selections from the flat top-k; this file holds the
// summaries, the per-row block positions and the map from compact selections
// back to token columns.
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

// One CTA (128 threads, thread = dim d) per item: the mean of the block's keys.
__global__ void __launch_bounds__(kDi) block_summary_kernel(BlockSumArgs a) {
  pdl_wait();
  const int i = blockIdx.x, d = threadIdx.x;
  const int s = a.item_seq[i];
  if (s < 0 || s >= a.n_seq) {
    if (d == 0) flag_error(a.err, LSA_DEVERR_SEQ);
    return;
  }
  const int64_t base = a.k_off[s], len = a.k_off[s + 1] - base;
  const int64_t bbase = a.blk_off[s], nb = a.blk_off[s + 1] - bbase;
  const int64_t b = a.item_blk[i];
  const int64_t t0 = b * a.block, t1 = min64(t0 + a.block, len);
  if (b < 0 || b >= nb || t0 >= len) {
    if (d == 0) flag_error(a.err, LSA_DEVERR_POS);
    return;
  }
  const uint16_t* __restrict__ k = a.k_idx + (base + t0) * kDi + d;
  // fp64 sum: exact for up to 1024 bf16 terms spanning fewer than 35 binades, so
  // the mean is the correctly rounded fp64 quotient before the bf16 rounding
  double sum = 0.0;
  for (int64_t t = 0; t < t1 - t0; ++t) sum += (double)__uint_as_float((uint32_t)__ldg(k + t * kDi) << 16);
  a.k_blk[(bbase + b) * kDi + d] = f64_to_bf16_rne(sum / (double)(t1 - t0));
  pdl_trigger();
}

__global__ void hier_prep_kernel(const int32_t* __restrict__ pos, int n_rows, int block, int32_t* __restrict__ pos_b) {
  pdl_wait();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r < n_rows) {
    const int p = pos[r];
    pos_b[r] = p >= 0 ? p / block : -1;
  }
  pdl_trigger();
}

// One CTA per row.
__global__ void __launch_bounds__(256) hier_map_kernel(const int32_t* __restrict__ pos,
                                                       const int32_t* __restrict__ sorted, int kb, int block,
                                                       int topk, int32_t* __restrict__ idx,
                                                       int32_t* __restrict__ count) {
  pdl_wait();
  const int r = blockIdx.x;
  const int p = pos[r];
  int32_t* __restrict__ ir = idx + (int64_t)r * topk;
  if (p < 0 || p + 1 <= topk) {  // dense row (or an invalid one, flagged upstream: empty)
    const int n = p < 0 ? 0 : p + 1;
    for (int i = threadIdx.x; i < topk; i += blockDim.x) ir[i] = i < n ? i : -1;
    if (threadIdx.x == 0) count[r] = n;
  } else {
    const int n = count[r];
    const int32_t* __restrict__ sr = sorted + (int64_t)r * kb;
    for (int i = threadIdx.x; i < topk; i += blockDim.x) {
      const int c = ir[i];
      if (i < n && c >= 0) ir[i] = sr[c / block] * block + c % block;
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_block_summaries(const BlockSumArgs& a, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  count_launches(1);
  return launch_pdl(block_summary_kernel, dim3(a.n_items), dim3(kDi), 0, st, a);
}

cudaError_t launch_hier_prep(const int32_t* pos, int n_rows, int block, int32_t* pos_b, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  count_launches(1);
  return launch_pdl(hier_prep_kernel, dim3((n_rows + 255) / 256), dim3(256), 0, st, pos, n_rows, block, pos_b);
}

cudaError_t launch_hier_map(const int32_t* pos, const int32_t* sorted, int kb, int block, int n_rows, int topk,
                            int32_t* idx, int32_t* count, cudaStream_t st) {
  if (n_rows <= 0) return cudaSuccess;
  count_launches(1);
  return launch_pdl(hier_map_kernel, dim3(n_rows), dim3(256), 0, st, pos, sorted, kb, block, topk, idx, count);
}

}  // namespace lsa
