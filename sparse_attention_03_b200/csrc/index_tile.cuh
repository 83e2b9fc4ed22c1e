// Key tiles of the streaming lightning indexer, shared by the decode indexer
// and the hierarchical fine stage: 16 keys per warp as the M dimension of
// mma.m16n8k16 (bf16 in, fp32 accumulate), the 32 index heads as four n8 tiles,
// the 128 dims as eight k16 steps, the contraction dimension permuted
// identically for keys and queries so that a lane's fragments of a key row are
// four contiguous 16-byte chunks; then the ReLU-weighted head sum.
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）" (q.k per index head, ReLU, head weights).
#pragma once

#include "common.cuh"

namespace lsa {
namespace idx {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kKeysPerWarpTile = 16;

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

}  // namespace idx
}  // namespace lsa
