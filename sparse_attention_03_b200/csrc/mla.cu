// Sparse absorbed-latent MLA over selected keys (decode and prefill rows).
//
// [Lite-Sparse] "架构总览": MLA in the kv-LoRA latent space, kv_lora_rank 512,
// qk_rope_head_dim 64, 32 heads; the absorbed query (embed_q) is dotted with
// whole 576-dim latent rows and the output is the 512-dim latent per head
// (unembed_out follows downstream).
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）": at decode the latent rows are
// gathered by the top-k indices; at prefill a sparse boolean mask keeps the
// same set. Both are computed here by gathering each row's selected keys, which
// gives exactly the masked result without touching unselected keys.
//
// Design. One CTA handles one (query row, split of its key list, sub-block).
// Latent rows are gathered by cp.async into a double-buffered shared-memory
// tile of 64 keys (1152-byte rows padded to 1168 so ldmatrix is conflict-free).
// S = Q K^T runs on mma.m16n8k16 with the 32 heads as M (2 tiles) and the keys
// split across 4 warps; the online softmax (base-2, max-subtracted) reduces
// across warps through shared memory; O += P V runs with the 512 value dims
// split across the warps (128 each, fp32 accumulators in registers). With more
// than one split per row the CTA writes an unnormalised partial (O, m, l) and a
// merge kernel combines the splits; with one split it writes bf16 output and lse
// directly. Gathered indices are bounds-checked against the row's visible keys.
#include "common.cuh"
#include "kernels.h"

namespace lsa {
namespace {

constexpr int kTK = 64;             // keys per tile
constexpr int kSRow = kDLat + 8;    // shared row stride (bf16): 1168 bytes
constexpr int kPRow = kTK + 8;      // P row stride (bf16): 144 bytes
constexpr int kMaxSplitKeys = 2048;
constexpr int kThreads = 128;
constexpr int kMaxSplits = 32;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

struct __align__(16) MlaSmem {
  uint16_t q[kH * kSRow];
  uint16_t k[2][kTK * kSRow];
  uint16_t p[kH * kPRow];
  float red[2][4][kH];
  int32_t list[kMaxSplitKeys];
};

struct Split {
  int n_split;
  int split_keys;
};

__global__ void __launch_bounds__(kThreads, 1) mla_kernel(MlaArgs a, Split sp, float* part_o,
                                                          float2* part_ml) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  MlaSmem& sm = *reinterpret_cast<MlaSmem*>(smem_raw);
  const int s = blockIdx.x, r = blockIdx.y, z = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;

  // ---- row geometry (clamped and flagged, never faulting) ----
  int64_t kbase = 0, nvis = 0;
  if (a.decode) {
    const int seq = a.seq_of_row ? a.seq_of_row[r] : r;
    if (seq < 0 || seq >= a.n_seq) {
      if (s == 0 && tid == 0) flag_error(a.err, LSA_DEVERR_SEQ);
    } else {
      kbase = a.k_off[seq];
      const int64_t klen = a.k_off[seq + 1] - kbase;
      nvis = klen;
      if (a.pos) {
        int64_t p1 = (int64_t)a.pos[r] + 1;
        if (p1 < 1 || p1 > klen) {
          if (s == 0 && tid == 0) flag_error(a.err, LSA_DEVERR_POS);
          p1 = max64(0, min(p1, klen));
        }
        nvis = p1;
      }
    }
  } else {
    int64_t p1 = (int64_t)a.pos[r] + 1;
    if (p1 < 1 || p1 > a.n_keys) {
      if (s == 0 && tid == 0) flag_error(a.err, LSA_DEVERR_POS);
      p1 = max64(0, min(p1, a.n_keys));
    }
    nvis = p1;
  }
  int64_t n_list = nvis;
  if (a.idx) {
    int c = a.count[r];
    if (c < 0 || c > a.topk) {
      if (s == 0 && tid == 0) flag_error(a.err, LSA_DEVERR_COUNT);
      c = max(0, min(c, a.topk));
    }
    n_list = c;
  }
  const int64_t b0 = (int64_t)s * sp.split_keys;
  const int nk = (int)max64(0, min64(sp.split_keys, n_list - b0));

  for (int i = tid; i < nk; i += kThreads) {
    int64_t key = a.idx ? (int64_t)a.idx[(int64_t)r * a.topk + b0 + i] : b0 + i;
    if (key < 0 || key >= nvis) {
      flag_error(a.err, LSA_DEVERR_INDEX);
      key = -1;
    }
    sm.list[i] = (int32_t)key;
  }
  const uint16_t* __restrict__ qg = a.q[z] + (int64_t)r * kH * kDLat;
  for (int c = tid; c < kH * (kDLat / 8); c += kThreads) {
    const int h = c / (kDLat / 8), col = c % (kDLat / 8);
    cp_async16(smem_u32(&sm.q[h * kSRow + col * 8]), qg + h * kDLat + col * 8, 16);
  }
  cp_async_commit();
  __syncthreads();

  const uint16_t* __restrict__ latb = a.lat[z] + kbase * kDLat;
  const int n_tiles = (nk + kTK - 1) / kTK;
  // Warp w gathers tile rows [16w, 16w+16): 16 x 72 16-byte chunks, 36 per lane,
  // consecutive lanes on consecutive chunks of a row.
  auto issue_tile = [&](int tt) {
    uint16_t* dst = sm.k[tt & 1];
#pragma unroll 4
    for (int u = 0; u < 36; ++u) {
      const int qd = lane + 32 * u;
      const int row = 16 * warp + qd / 72, col = qd % 72;
      const int slot = tt * kTK + row;
      const int key = slot < nk ? sm.list[slot] : -1;
      const uint16_t* src = key >= 0 ? latb + (int64_t)key * kDLat + col * 8 : a.lat[z];
      cp_async16(smem_u32(dst + row * kSRow + col * 8), src, key >= 0 ? 16 : 0);
    }
  };
  if (n_tiles > 0) issue_tile(0);
  cp_async_commit();

  const float scale_log2 = a.scale * kLog2e;
  float m_run[2][2], l_run[2][2];
  float o[2][16][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      m_run[mt][hf] = -INFINITY;
      l_run[mt][hf] = 0.f;
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) o[mt][nt][i] = 0.f;
  }

  for (int tt = 0; tt < n_tiles; ++tt) {
    if (tt + 1 < n_tiles) issue_tile(tt + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint16_t* kt = sm.k[tt & 1];

    // ---- S = Q K^T for keys 16w .. 16w+15 of the tile ----
    float sc[2][2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[mt][nt][i] = 0.f;
    const uint32_t qa0 = smem_u32(&sm.q[(lane & 15) * kSRow + 8 * (lane >> 4)]);
    const uint32_t qa1 = qa0 + 16 * kSRow * 2;
    const uint32_t kb0 =
        smem_u32(&kt[(16 * warp + (lane & 7) + 8 * (lane >> 4)) * kSRow + 8 * ((lane >> 3) & 1)]);
#pragma unroll 4
    for (int ks = 0; ks < kDLat / 16; ++ks) {
      uint32_t a0[4], a1[4], b[4];
      ldsm_x4(qa0 + ks * 32, a0[0], a0[1], a0[2], a0[3]);
      ldsm_x4(qa1 + ks * 32, a1[0], a1[1], a1[2], a1[3]);
      ldsm_x4(kb0 + ks * 32, b[0], b[1], b[2], b[3]);
      mma_16816(sc[0][0], a0[0], a0[1], a0[2], a0[3], b[0], b[1]);
      mma_16816(sc[0][1], a0[0], a0[1], a0[2], a0[3], b[2], b[3]);
      mma_16816(sc[1][0], a1[0], a1[1], a1[2], a1[3], b[0], b[1]);
      mma_16816(sc[1][1], a1[0], a1[1], a1[2], a1[3], b[2], b[3]);
    }

    // ---- online softmax (base 2) ----
    // sc[mt][nt][2*hf+e]: head 16mt+8hf+g, key 16w+8nt+2t+e.
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int slot = tt * kTK + 16 * warp + 8 * nt + 2 * t + e;
        const bool valid = slot < nk && sm.list[slot] >= 0;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            sc[mt][nt][2 * hf + e] = valid ? sc[mt][nt][2 * hf + e] * scale_log2 : -INFINITY;
      }
    float mx[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v = fmaxf(fmaxf(sc[mt][0][2 * hf], sc[mt][0][2 * hf + 1]),
                        fmaxf(sc[mt][1][2 * hf], sc[mt][1][2 * hf + 1]));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
        if (t == 0) sm.red[0][warp][16 * mt + 8 * hf + g] = v;
      }
    __syncthreads();
    float alpha[2][2], m_use[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int head = 16 * mt + 8 * hf + g;
        const float tmax = fmaxf(fmaxf(sm.red[0][0][head], sm.red[0][1][head]),
                                 fmaxf(sm.red[0][2][head], sm.red[0][3][head]));
        const float m_new = fmaxf(m_run[mt][hf], tmax);
        m_use[mt][hf] = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[mt][hf] = exp2f(m_run[mt][hf] - m_use[mt][hf]);
        m_run[mt][hf] = m_new;
        mx[mt][hf] = 0.f;
      }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float p0 = exp2f(sc[mt][nt][2 * hf] - m_use[mt][hf]);
          const float p1 = exp2f(sc[mt][nt][2 * hf + 1] - m_use[mt][hf]);
          mx[mt][hf] += p0 + p1;
          const int head = 16 * mt + 8 * hf + g;
          *reinterpret_cast<uint32_t*>(&sm.p[head * kPRow + 16 * warp + 8 * nt + 2 * t]) =
              pack_bf16x2(p0, p1);
        }
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v = mx[mt][hf];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        if (t == 0) sm.red[1][warp][16 * mt + 8 * hf + g] = v;
      }
    __syncthreads();
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int head = 16 * mt + 8 * hf + g;
        const float tsum = (sm.red[1][0][head] + sm.red[1][1][head]) +
                           (sm.red[1][2][head] + sm.red[1][3][head]);
        l_run[mt][hf] = l_run[mt][hf] * alpha[mt][hf] + tsum;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[mt][nt][2 * hf] *= alpha[mt][hf];
          o[mt][nt][2 * hf + 1] *= alpha[mt][hf];
        }
      }

    // ---- O += P V for value dims 128w .. 128w+127 ----
    const uint32_t pa0 = smem_u32(&sm.p[(lane & 15) * kPRow + 8 * (lane >> 4)]);
    const uint32_t pa1 = pa0 + 16 * kPRow * 2;
    const uint32_t vb0 = smem_u32(
        &kt[((lane & 7) + 8 * ((lane >> 3) & 1)) * kSRow + 128 * warp + 8 * (lane >> 4)]);
#pragma unroll
    for (int kk = 0; kk < kTK / 16; ++kk) {
      uint32_t p0[4], p1[4];
      ldsm_x4(pa0 + kk * 32, p0[0], p0[1], p0[2], p0[3]);
      ldsm_x4(pa1 + kk * 32, p1[0], p1[1], p1[2], p1[3]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t v[4];
        ldsm_x4_t(vb0 + (kk * 16 * kSRow + 16 * np) * 2, v[0], v[1], v[2], v[3]);
        mma_16816(o[0][2 * np], p0[0], p0[1], p0[2], p0[3], v[0], v[1]);
        mma_16816(o[0][2 * np + 1], p0[0], p0[1], p0[2], p0[3], v[2], v[3]);
        mma_16816(o[1][2 * np], p1[0], p1[1], p1[2], p1[3], v[0], v[1]);
        mma_16816(o[1][2 * np + 1], p1[0], p1[1], p1[2], p1[3], v[2], v[3]);
      }
    }
    __syncthreads();  // buffer tt&1, P and red are rewritten next iteration
  }
  cp_async_wait<0>();

  // ---- epilogue ----
  if (sp.n_split == 1) {
    uint16_t* __restrict__ og = a.out[z] + (int64_t)r * kH * kDV;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int head = 16 * mt + 8 * hf + g;
        const float l = l_run[mt][hf];
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          const int d = 128 * warp + 8 * nt + 2 * t;
          *reinterpret_cast<uint32_t*>(&og[head * kDV + d]) =
              pack_bf16x2(o[mt][nt][2 * hf] * inv, o[mt][nt][2 * hf + 1] * inv);
        }
        if (a.lse[z] && warp == 0 && t == 0)
          a.lse[z][(int64_t)r * kH + head] =
              l > 0.f ? (m_run[mt][hf] + log2f(l)) * kLn2 : -INFINITY;
      }
  } else {
    const int64_t base = ((int64_t)z * a.n_rows + r) * sp.n_split + s;
    float* __restrict__ po = part_o + base * kH * kDV;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int head = 16 * mt + 8 * hf + g;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          const int d = 128 * warp + 8 * nt + 2 * t;
          *reinterpret_cast<float2*>(&po[head * kDV + d]) =
              make_float2(o[mt][nt][2 * hf], o[mt][nt][2 * hf + 1]);
        }
        if (warp == 0 && t == 0) part_ml[base * kH + head] = make_float2(m_run[mt][hf], l_run[mt][hf]);
      }
  }
}

__global__ void __launch_bounds__(256) mla_merge_kernel(MlaArgs a, Split sp, const float* part_o,
                                                        const float2* part_ml) {
  __shared__ float wgt[kMaxSplits][kH];
  __shared__ float inv_l[kH];
  const int r = blockIdx.x, z = blockIdx.y, tid = threadIdx.x;
  const int64_t base = ((int64_t)z * a.n_rows + r) * sp.n_split;
  if (tid < kH) {
    float M = -INFINITY;
    for (int s = 0; s < sp.n_split; ++s) M = fmaxf(M, part_ml[(base + s) * kH + tid].x);
    float L = 0.f;
    for (int s = 0; s < sp.n_split; ++s) {
      const float2 ml = part_ml[(base + s) * kH + tid];
      const float wv = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
      wgt[s][tid] = wv;
      L += wv * ml.y;
    }
    inv_l[tid] = L > 0.f ? 1.f / L : 0.f;
    if (a.lse[z]) a.lse[z][(int64_t)r * kH + tid] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
  }
  __syncthreads();
  uint16_t* __restrict__ og = a.out[z] + (int64_t)r * kH * kDV;
  for (int e = tid * 4; e < kH * kDV; e += 256 * 4) {
    const int head = e / kDV;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < sp.n_split; ++s) {
      const float4 v = *reinterpret_cast<const float4*>(part_o + (base + s) * kH * kDV + e);
      const float wv = wgt[s][head];
      acc.x = fmaf(wv, v.x, acc.x);
      acc.y = fmaf(wv, v.y, acc.y);
      acc.z = fmaf(wv, v.z, acc.z);
      acc.w = fmaf(wv, v.w, acc.w);
    }
    const float il = inv_l[head];
    uint2 pk;
    pk.x = pack_bf16x2(acc.x * il, acc.y * il);
    pk.y = pack_bf16x2(acc.z * il, acc.w * il);
    *reinterpret_cast<uint2*>(og + e) = pk;
  }
}

}  // namespace

size_t mla_ws_bytes(int n_rows, int cli, int n_split) {
  if (n_split <= 1) return 0;
  const size_t per = (size_t)kH * kDV * sizeof(float) + (size_t)kH * sizeof(float2);
  return (size_t)n_rows * cli * n_split * per + 256;
}

int mla_choose_splits(int n_rows, int cli, int64_t max_list) {
  // Enough CTAs to cover the SMs about twice, splits of at least 256 keys,
  // each split at most 2048 keys (the shared-memory index list).
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t work = (int64_t)n_rows * cli;
  int64_t by_len = (max_list + 255) / 256;
  int64_t want = (2 * sms + work - 1) / max64(work, 1);
  int64_t n = min(by_len, want);
  const int64_t min_for_list = (max_list + kMaxSplitKeys - 1) / kMaxSplitKeys;
  n = max(n, min_for_list);
  n = max64(1, min64(n, kMaxSplits));
  return (int)n;
}

cudaError_t launch_mla(const MlaArgs& a, cudaStream_t st) {
  if (a.n_rows <= 0) return cudaSuccess;
  int n_split = mla_choose_splits(a.n_rows, a.cli, a.max_list);
  const int64_t min_for_list = (a.max_list + kMaxSplitKeys - 1) / kMaxSplitKeys;
  // Shrink split-K to what the workspace holds (never below what the list needs).
  while (n_split > 1 && n_split > min_for_list && mla_ws_bytes(a.n_rows, a.cli, n_split) > a.ws_bytes)
    --n_split;
  if (n_split > 1 && mla_ws_bytes(a.n_rows, a.cli, n_split) > a.ws_bytes) return cudaErrorInvalidValue;
  Split sp;
  sp.n_split = n_split;
  sp.split_keys = (int)(((a.max_list + n_split - 1) / n_split + kTK - 1) / kTK * kTK);
  if (sp.split_keys > kMaxSplitKeys) return cudaErrorInvalidValue;
  float* part_o = nullptr;
  float2* part_ml = nullptr;
  if (n_split > 1) {
    uintptr_t p = (reinterpret_cast<uintptr_t>(a.ws) + 255) & ~uintptr_t(255);
    part_o = reinterpret_cast<float*>(p);
    part_ml = reinterpret_cast<float2*>(part_o + (size_t)a.n_rows * a.cli * n_split * kH * kDV);
  }
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(MlaSmem));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  for (int row0 = 0; row0 < a.n_rows; row0 += 65535) {
    MlaArgs b = a;
    const int nr = min(65535, a.n_rows - row0);
    // Row offsets are folded into the pointers of this chunk.
    b.n_rows = a.n_rows;
    if (row0 > 0) {
      // rows beyond 65535 are handled by shifting every per-row pointer
      for (int z = 0; z < a.cli; ++z) {
        b.q[z] = a.q[z] + (int64_t)row0 * kH * kDLat;
        b.out[z] = a.out[z] + (int64_t)row0 * kH * kDV;
        b.lse[z] = a.lse[z] ? a.lse[z] + (int64_t)row0 * kH : nullptr;
      }
      if (b.seq_of_row) b.seq_of_row += row0;
      if (b.pos) b.pos += row0;
      if (b.idx) b.idx += (int64_t)row0 * a.topk;
      if (b.count) b.count += row0;
    }
    b.n_rows = nr;
    // decode without seq_of_row maps row -> sequence by row number: keep that
    // mapping across chunks by offsetting k_off.
    if (b.decode && !a.seq_of_row && row0 > 0) {
      b.k_off = a.k_off + row0;
      b.n_seq = a.n_seq - row0;
    }
    mla_kernel<<<dim3(n_split, nr, a.cli), kThreads, sizeof(MlaSmem), st>>>(b, sp, part_o, part_ml);
    if (n_split > 1) mla_merge_kernel<<<dim3(nr, a.cli), 256, 0, st>>>(b, sp, part_o, part_ml);
    count_launches(n_split > 1 ? 2 : 1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace lsa
