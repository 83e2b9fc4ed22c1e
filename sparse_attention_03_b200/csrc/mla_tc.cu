// Sparse absorbed-latent MLA on the 5th-generation tensor cores (tcgen05):
// keys (and value dims) as the M dimension, the 32 heads as N.
//
// [Lite-Sparse] "架构总览": absorbed MLA over 576-dim latent rows (512 c_kv +
// 64 rope), 32 heads, values = the first 512 dims.
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）": at decode the latent rows are
// gathered by the top-k indices; at prefill each row's selected set is the
// sparse mask. Both are computed by gathering each row's selected keys.
//
// Design. With 32 heads a heads-as-M MMA is half padding, and tcgen05 then
// runs no faster than the legacy mma.sync path; with keys as M (128 keys a
// tile) and heads as N = 32 every MMA row is useful. One CTA handles one (query
// row, split of its key list, sub-block):
//   * S^T = K Q^T: M = 128 keys, N = 32 heads, K = 576 (36 MMAs) into one of two
//     32-column fp32 accumulators in tensor memory (thread = key, column = head).
//   * O^T += V^T P^T: M = 128 value dims (four blocks for 512), N = 32 heads,
//     K = 128 keys (8 MMAs a block) into 4 x 32 columns of tensor memory.
//   * The 128-key tile does not fit twice in shared memory (144 KB), so the
//     keys stream through a ring of five 32 KB slots, two 64-dim chunks each,
//     gathered by TMA (tile::gather4, 128-byte swizzle): five slots for the
//     logits (576 dims, the last half full), then the first 512 dims of the same
//     keys again (an L2 hit) for the values. The same bytes are the K-major A
//     operand of S^T and the MN-major A operand of O^T.
//   * Softmax: four warps, one key per thread and all 32 heads in registers. A
//     per-head reference max is fixed on the first tile and moves only when a
//     tile's logit exceeds it by more than 8 (base 2), so P stays below 2^8 and
//     O^T is rescaled rarely; the row sums accumulate per thread and are reduced
//     once at the end. P^T (bf16, [head][key], swizzled) goes to shared memory.
//   * Warp 0 issues TMA, warp 1 allocates tensor memory and issues the MMAs
//     (logits of tile t+1 before the values of tile t, so the softmax of one
//     tile overlaps the tensor core), warps 2-5 run the softmax and the epilogue.
// Every wait is bounded; on timeout the CTA raises an error flag and stops.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "launch.h"
#include "mla_common.cuh"
#include "tc.cuh"

namespace lsa {
namespace {

constexpr int kT = 128;                      // keys per tile
constexpr int kSlots = 5;                    // ring slots
constexpr uint32_t kChunk = 128 * 128;       // 16 KB: 128 keys x 64 dims bf16
constexpr uint32_t kSlotBytes = 2 * kChunk;  // two 64-dim chunks
constexpr int kQkUnits = 5;                  // 9 chunks of logits dims: 4 full slots + 1 half
constexpr int kPvUnits = 4;                  // 8 chunks of value dims
constexpr uint32_t kQChunk = 32 * 128;       // 4 KB: 32 heads x 64 dims
constexpr uint32_t kPBlock = 32 * 128;       // 4 KB: 32 heads x 64 keys
constexpr int kTcThreads = 6 * 32;
constexpr int kSmxThreads = 128;
constexpr int kTmemCols = 256;               // S^T x2 (64 cols) + O^T (128 cols)
constexpr uint32_t kOCol = 64;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kRescaleAt = 8.f;            // base-2 headroom before O^T is rescaled

// kind::f16, A = B = bf16, D = fp32, M = 128, N = 32; A K-major (logits) or
// MN-major (values), B K-major.
constexpr uint32_t kIdescQK = (1u << 4) | (1u << 7) | (1u << 10) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescQK | (1u << 15);

struct __align__(1024) TcSmem {
  uint8_t ring[kSlots][kSlotBytes];   // gathered key chunks, swizzled
  uint8_t q[9 * kQChunk];             // Q: [dim chunk][32 heads x 128 B], swizzled
  uint8_t p[2][2 * kPBlock];          // P^T: [key block][32 heads x 128 B], swizzled
  int32_t list[kMaxTopk];             // this split's validated keys (-1 masked)
  float red[4][kH];
  uint64_t full[kSlots], empty[kSlots], sfull[2], sfree[2], pfull[2], pfree[2], qbar;
  uint32_t tmem_base;
  int abort_flag;
};

struct TcSplit {
  int n_split;
  int list_tiles;  // 128-key tiles of the longest list (the split boundaries)
};

__device__ __forceinline__ void gather4(void* dst, const CUtensorMap* map, int x, int y0, int y1, int y2, int y3,
                                        uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier 1 over the four softmax warps, with an OR of a predicate.
__device__ __forceinline__ bool smx_sync_or(bool v) {
  uint32_t out;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(out)
      : "r"(v ? 1u : 0u), "n"(kSmxThreads)
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void smx_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(kSmxThreads) : "memory"); }

// Per-head maximum over the 128 softmax threads (one key each) of x[32].
__device__ __forceinline__ void head_max(const float (&x)[kH], float (&red)[4][kH], int sw, int lane,
                                         float (&out)[kH]) {
#pragma unroll
  for (int h = 0; h < kH; ++h) {
    float v = x[h];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == h) red[sw][h] = v;
  }
  smx_sync();
#pragma unroll
  for (int h = 0; h < kH; ++h) out[h] = fmaxf(fmaxf(red[0][h], red[1][h]), fmaxf(red[2][h], red[3][h]));
  smx_sync();
}

__device__ __forceinline__ void head_sum(const float (&x)[kH], float (&red)[4][kH], int sw, int lane,
                                         float (&out)[kH]) {
#pragma unroll
  for (int h = 0; h < kH; ++h) {
    float v = x[h];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == h) red[sw][h] = v;
  }
  smx_sync();
#pragma unroll
  for (int h = 0; h < kH; ++h) out[h] = (red[0][h] + red[1][h]) + (red[2][h] + red[3][h]);
  smx_sync();
}

// Both the producer and the MMA issuer walk the same unit sequence: the logits
// of tile g (kQkUnits slots), then the values of tile g-1 (kPvUnits slots); the
// values of the last tile close it. The k-th unit used sits in slot k % kSlots.
template <class F>
__device__ __forceinline__ void walk_units(int n_tiles, F&& f) {
  int k = 0;
  for (int g = 0; g <= n_tiles; ++g) {
    if (g < n_tiles)
      for (int u = 0; u < kQkUnits; ++u)
        if (!f(false, g, u, k++)) return;
    if (g >= 1)
      for (int u = 0; u < kPvUnits; ++u)
        if (!f(true, g - 1, u, k++)) return;
  }
}

__global__ void __launch_bounds__(kTcThreads, 1)
    mla_tc_kernel(const __grid_constant__ CUtensorMap map_lat0, const __grid_constant__ CUtensorMap map_lat1,
                  const __grid_constant__ CUtensorMap map_q0, const __grid_constant__ CUtensorMap map_q1,
                  MlaArgs a, TcSplit sp, float* part_o, float2* part_ml) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {  // swizzled operands need 1024-byte aligned bases
    if (threadIdx.x == 0) flag_error(a.err, LSA_DEVERR_TIMEOUT);
    return;
  }
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw);
  const int s = blockIdx.x, r = blockIdx.y, z = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const CUtensorMap* map_lat = z == 0 ? &map_lat0 : &map_lat1;
  const CUtensorMap* map_q = z == 0 ? &map_q0 : &map_q1;
  if (tid == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.sfree[i], 4);
      mbar_init(&sm.pfull[i], 4);
      mbar_init(&sm.pfree[i], 1);
    }
    mbar_init(&sm.qbar, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
  }
  pdl_wait();

  // This split's keys: whole 128-key tiles of the longest list, clipped to the row's own.
  const int64_t t_lo = (int64_t)sp.list_tiles * s / sp.n_split;
  const int64_t t_hi = (int64_t)sp.list_tiles * (s + 1) / sp.n_split;
  const int64_t b0 = t_lo * kT;
  const int cap = (int)((t_hi - t_lo) * kT);
  const RowGeom geo = row_geometry(a, r, s == 0 && tid == 0);
  const int nk = (int)max64(0, min64((int64_t)cap, geo.n_list - b0));
  const int n_tiles = (nk + kT - 1) / kT;
  const int32_t* __restrict__ irow = a.idx ? a.idx + (int64_t)r * a.topk + b0 : nullptr;
  // With an index list the split holds at most topk <= kMaxTopk keys; a dense
  // row's keys are b0 + slot and need no list.
  if (irow)
    for (int i = tid; i < nk; i += kTcThreads) {
      int64_t key = __ldg(irow + i);
      if (key < 0 || key >= geo.nvis) {
        flag_error(a.err, LSA_DEVERR_INDEX);
        key = -1;
      }
      sm.list[i] = (int32_t)key;
    }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();  // barriers initialised, key list and tensor memory ready
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  // key slot -> absolute latent row (a masked slot loads the sequence's first row;
  // its weight is exactly 0)
  auto key_of = [&](int slot) -> int {
    if (slot >= nk) return -1;
    return irow ? sm.list[slot] : (int)(b0 + slot);
  };

  if (warp == 0) {
    // ================= TMA producer =================
    if (n_tiles > 0) {
      if (lane == 0) {
        mbar_expect_tx(&sm.qbar, 9 * kQChunk);
        for (int c = 0; c < 9; ++c) tma_load_2d(sm.q + c * kQChunk, map_q, 64 * c, r * kH, &sm.qbar);
      }
      const int base_row = (int)geo.kbase;
      walk_units(n_tiles, [&](bool pv, int tile, int u, int k) -> bool {
        const int slot = k % kSlots;
        if (k >= kSlots && !mbar_wait(&sm.empty[slot], ((k / kSlots) - 1) & 1, abort_flag)) return false;
        const int n_chunks = (!pv && u == kQkUnits - 1) ? 1 : 2;
        if (lane == 0) mbar_expect_tx(&sm.full[slot], n_chunks * kChunk);
        __syncwarp();
        // lane = a group of 4 keys; one gather4 per 64-dim chunk
        int rows[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int key = key_of(tile * kT + 4 * lane + q);
          rows[q] = base_row + (key >= 0 ? key : 0);
        }
        for (int c = 0; c < n_chunks; ++c)
          gather4(sm.ring[slot] + c * kChunk + lane * 512, map_lat, 64 * (2 * u + c), rows[0], rows[1], rows[2],
                  rows[3], &sm.full[slot]);
        return true;
      });
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0 && n_tiles > 0) {
      bool ok = mbar_wait(&sm.qbar, 0, abort_flag);
      const uint32_t q_base = smem_u32(sm.q);
      if (ok)
        walk_units(n_tiles, [&](bool pv, int tile, int u, int k) -> bool {
          const int slot = k % kSlots;
          const int b = tile & 1;
          if (!pv && u == 0 && tile >= 2 && !mbar_wait(&sm.sfree[b], ((tile - 2) >> 1) & 1, abort_flag))
            return false;
          if (pv && u == 0 && !mbar_wait(&sm.pfull[b], (tile >> 1) & 1, abort_flag)) return false;
          if (!mbar_wait(&sm.full[slot], (k / kSlots) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t ring = smem_u32(sm.ring[slot]);
          if (!pv) {
            const int n_chunks = (u == kQkUnits - 1) ? 1 : 2;
            for (int c = 0; c < n_chunks; ++c) {
              const int dimc = 2 * u + c;
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                umma_f16(tmem + 32 * b, sw128_desc(ring + c * kChunk + ks * 32),
                         sw128_desc(q_base + dimc * kQChunk + ks * 32), kIdescQK, (dimc > 0 || ks > 0) ? 1u : 0u);
            }
            umma_commit(&sm.empty[slot]);
            if (u == kQkUnits - 1) umma_commit(&sm.sfull[b]);
          } else {
            const uint32_t p_base = smem_u32(sm.p[b]);
#pragma unroll
            for (int ks = 0; ks < kT / 16; ++ks)
              umma_f16(tmem + kOCol + 32 * u, sw128_mn_desc(ring + ks * 2048, kChunk),
                       sw128_desc(p_base + (ks >> 2) * kPBlock + (ks & 3) * 32), kIdescPV,
                       (tile > 0 || ks > 0) ? 1u : 0u);
            umma_commit(&sm.empty[slot]);
            if (u == kPvUnits - 1) umma_commit(&sm.pfree[b]);
          }
          return true;
        });
    }
  } else {
    // ================= softmax and epilogue (warps 2..5) =================
    // Thread = tensor-memory lane = key slot i of a tile (logits) and value dim
    // 128m + i of block m (output); a warp may touch lanes 32 (warp % 4) .. +31.
    const int sw = warp - 2;
    const int i = 32 * (warp & 3) + lane;
    const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
    const float scale_log2 = a.scale * kLog2e;
    float m_ref[kH], l_part[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h) {
      m_ref[h] = -INFINITY;
      l_part[h] = 0.f;
    }
    // a lane waits, the warp follows (tensor-memory loads are warp-wide); after
    // an abort every wait returns at once, so the four warps stay in step
    auto warp_wait = [&](uint64_t* bar, uint32_t parity) {
      if (lane == 0) mbar_wait(bar, parity, abort_flag);
      __syncwarp();
    };
    for (int t = 0; t < n_tiles; ++t) {
      const int b = t & 1;
      warp_wait(&sm.sfull[b], (t >> 1) & 1);
      tc_fence_after();
      float x[kH];
      tmem_ld32(tmem + lane_addr + 32 * b, x);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sfree[b]);
      const bool valid = key_of(t * kT + i) >= 0;
#pragma unroll
      for (int h = 0; h < kH; ++h) x[h] = valid ? x[h] * scale_log2 : -INFINITY;
      bool need = t == 0;
      if (t > 0) {
        bool mine = false;
#pragma unroll
        for (int h = 0; h < kH; ++h) mine |= x[h] > m_ref[h] + kRescaleAt;
        need = smx_sync_or(mine);
      }
      if (need) {
        float tmax[kH];
        head_max(x, sm.red, sw, lane, tmax);
        float alpha[kH];
#pragma unroll
        for (int h = 0; h < kH; ++h) {
          const float mn = fmaxf(m_ref[h], tmax[h]);
          alpha[h] = mn == -INFINITY ? 1.f : exp2f(m_ref[h] - mn);
          m_ref[h] = mn;
          l_part[h] *= alpha[h];
        }
        if (t > 0) {
          // O^T holds the values of tiles < t-1 or t-1 complete: wait for tile t-1's, then rescale
          warp_wait(&sm.pfree[(t - 1) & 1], ((t - 1) >> 1) & 1);
          tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < kPvUnits; ++m) {
            float o[32];
            tmem_ld32(tmem + lane_addr + kOCol + 32 * m, o);
#pragma unroll
            for (int h = 0; h < kH; ++h) o[h] *= alpha[h];
            tmem_st32(tmem + lane_addr + kOCol + 32 * m, o);
          }
          tc_fence_before();
        }
      }
      // P^T buffer b was last read by the values of tile t-2
      if (t >= 2) warp_wait(&sm.pfree[b], ((t - 2) >> 1) & 1);
      uint8_t* pb = sm.p[b] + (i >> 6) * kPBlock;
      const int kk = i & 63;
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        const float mu = m_ref[h] == -INFINITY ? 0.f : m_ref[h];
        const float pv = exp2f(x[h] - mu);
        l_part[h] += pv;
        *reinterpret_cast<uint16_t*>(pb + h * 128 + (((kk >> 3) ^ (h & 7)) << 4) + (kk & 7) * 2) =
            f32_to_bf16_rne(pv);
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.pfull[b]);
    }
    pdl_trigger();

    // ---- epilogue ----
    float l[kH];
    head_sum(l_part, sm.red, sw, lane, l);
    const bool any = n_tiles > 0;
    if (any) {
      warp_wait(&sm.pfree[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1);
      tc_fence_after();
    }
    if (tid == 64 && *abort_flag) flag_error(a.err, LSA_DEVERR_TIMEOUT);
    const int64_t base = ((int64_t)z * a.n_rows + r) * sp.n_split + s;
#pragma unroll 1
    for (int m = 0; m < kPvUnits; ++m) {
      float o[32];
      if (any) {
        tmem_ld32(tmem + lane_addr + kOCol + 32 * m, o);
      } else {
#pragma unroll
        for (int h = 0; h < kH; ++h) o[h] = 0.f;
      }
      const int d = 128 * m + i;
      if (sp.n_split == 1) {
        uint16_t* __restrict__ og = a.out[z] + (int64_t)r * kH * kDV + d;
#pragma unroll
        for (int h = 0; h < kH; ++h) {
          const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
          og[h * kDV] = f32_to_bf16_rne(o[h] * inv);
        }
      } else {
        float* __restrict__ po = part_o + base * kH * kDV + d;
#pragma unroll
        for (int h = 0; h < kH; ++h) po[h * kDV] = o[h];
      }
    }
    if (i < kH) {
      float mh = 0.f, lh = 0.f;
#pragma unroll
      for (int h = 0; h < kH; ++h)
        if (h == i) {
          mh = m_ref[h];
          lh = l[h];
        }
      if (sp.n_split == 1) {
        if (a.lse[z]) a.lse[z][(int64_t)r * kH + i] = lh > 0.f ? (mh + log2f(lh)) * kLn2 : -INFINITY;
      } else {
        part_ml[base * kH + i] = make_float2(mh, lh);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

}  // namespace

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tc_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 map over [rows, 576] (1152-byte rows) with a box of box_rows x 64 and
// 128-byte swizzle. Coordinates past `rows` read zeros and never touch memory.
bool latent_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = tc_encode_fn();
  if (!fn || rows == 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDLat, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDLat * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool mla_tc_supported() { return tc_encode_fn() != nullptr; }

size_t mla_tc_smem_bytes() { return sizeof(TcSmem); }

// One chunk of at most 65535 rows (the caller shifts the per-row pointers).
// `lat_rows` bounds the latent rows a key may address (the tensor maps' extent).
cudaError_t launch_mla_tc_chunk(const MlaArgs& b, int n_split, int64_t max_list, int64_t lat_rows, float* part_o,
                                float2* part_ml, cudaStream_t st) {
  CUtensorMap ml[2], mq[2];
  for (int z = 0; z < 2; ++z) {
    const int zz = z < b.cli ? z : 0;
    if (!latent_map(&ml[z], b.lat[zz], (uint64_t)lat_rows, 1)) return cudaErrorInvalidValue;
    if (!latent_map(&mq[z], b.q[zz], (uint64_t)b.n_rows * kH, 32)) return cudaErrorInvalidValue;
  }
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(TcSmem));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  TcSplit sp;
  sp.n_split = n_split;
  const int64_t list = b.idx ? min64(max_list, (int64_t)min(b.topk, kMaxTopk)) : max_list;
  sp.list_tiles = (int)((list + kT - 1) / kT);
  return launch_pdl(mla_tc_kernel, dim3(n_split, b.n_rows, b.cli), dim3(kTcThreads), sizeof(TcSmem), st, ml[0],
                    ml[1], mq[0], mq[1], b, sp, part_o, part_ml);
}

}  // namespace lsa
