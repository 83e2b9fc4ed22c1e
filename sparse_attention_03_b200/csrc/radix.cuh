// Radix-select helpers shared by the top-k kernels and the indexer epilogue.
#pragma once

#include "common.cuh"

namespace lsa {

constexpr int kBins = 2048;  // 11-bit digits

// For a histogram h[0..BINS) and a budget `need`, finds the bin d such that
// (count in bins above d) < need <= (count in bins >= d). Block-wide; every
// thread returns the same answer.
template <int THREADS, int BINS = kBins>
__device__ void find_threshold(const uint32_t* h, uint32_t need, int& bin_out,
                               uint32_t& above_out, int* s_bin, uint32_t* s_above,
                               uint32_t* s_warp) {
  constexpr int PER = BINS / THREADS;
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


// The rest of the select inside the threshold bin. The candidates' low 53 bits
// (the 21 key bits below the top 11, then the bit-inverted column index) are
// unique, so a radix select from the top, 11 bits a level, ends with exactly
// `need` values v with (v >> (53 - decided)) >= prefix. It stops as soon as one
// bin holds exactly what is still needed. for_each(f) must call f(v53, column)
// for every candidate (each thread a share of them); every candidate must carry
// the top `decided0` bits `prefix0` (0 and 0 when nothing is decided yet).
// Block-wide.
template <int THREADS, class ForEach>
__device__ void radix_levels(ForEach&& for_each, uint32_t need, uint32_t* h, int* s_bin, uint32_t* s_above,
                             uint32_t* s_warp, uint64_t& prefix, int& decided, uint64_t prefix0 = 0,
                             int decided0 = 0) {
  prefix = prefix0;
  decided = decided0;
  while (decided < 53) {
    const int wdt = min(11, 53 - decided);
    const int shift = 53 - decided - wdt;
    for (int i = threadIdx.x; i < kBins; i += THREADS) h[i] = 0;
    __syncthreads();
    const uint64_t pf = prefix;
    const int dc = decided;
    for_each([&](uint64_t v, int64_t) {
      if ((v >> (53 - dc)) == pf) atomicAdd(&h[(uint32_t)(v >> shift) & ((1u << wdt) - 1u)], 1u);
    });
    __syncthreads();
    int d;
    uint32_t above;
    find_threshold<THREADS>(h, need, d, above, s_bin, s_above, s_warp);
    const uint32_t cnt = h[d];
    need -= above;
    prefix = (prefix << wdt) | (uint64_t)d;
    decided += wdt;
    __syncthreads();
    if (cnt == need) break;  // the whole bin is taken
  }
}

}  // namespace lsa
