// Lightning indexer, prefill form: a dense contraction on the 5th-generation
// tensor cores (tcgen05 MMA, accumulators in tensor memory, operands by TMA).
//
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）": per index head q.k, ReLU, then the
// head-weighted sum; sink and local-window columns forced to +inf.
// [Lite-Sparse] "预填充优化": the ReLU-weighted head sum is an epilogue on the
// q k^T product that never writes the per-head [tokens x heads x keys] tensor.
//
// Design. One CTA owns a block of 16 query rows (512 = 16 x 32 (token, head)
// rows of the B operand, 128 KB of shared memory, loaded once by TMA) and a run
// of 128-key tiles of the one sequence. For each key tile (A operand: 128 keys
// x 128 dims bf16, 32 KB, TMA with 128-byte swizzle, 3-stage ring) one thread
// issues two M=128 x N=256 x K=128 MMAs (8 instructions of K=16 each) into two
// 256-column fp32 accumulators in tensor memory: tokens 0-7 and tokens 8-15.
// Eight epilogue warps read the accumulators with tcgen05.ld (a thread = one key,
// 32 consecutive columns = the 32 heads of one token), apply ReLU and the head
// weights in registers, mask/force and store one fp32 score per (token, key);
// a warp's 32 lanes are 32 consecutive keys, so each store is a 128-byte line.
// A warp loads its 4 tokens x 32 heads of an accumulator in one round (one
// wait) and releases the accumulator before the math and the stores, so the
// tensor core refills it while the epilogue finishes; while the epilogue drains
// one accumulator the tensor core fills the other.
// Warp 0 issues TMA, warp 1 allocates tensor memory and issues MMAs, warps 2-9
// run the epilogue. Every mbarrier wait is bounded: on timeout the CTA raises an
// error flag, stops, and still frees its tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "launch.h"
#include "tc.cuh"

namespace lsa {
namespace {

constexpr int kRowsPerBlock = 16;                 // query rows per CTA
constexpr int kBRows = kRowsPerBlock * kHi;       // 512 (token, head) rows
constexpr int kTileKeys = 128;
constexpr int kStages = 3;
constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;    // 320
constexpr uint32_t kATileBytes = kTileKeys * kDi * 2;    // 32 KB
constexpr uint32_t kAHalfBytes = kATileBytes / 2;         // 16 KB (64 dims)
constexpr uint32_t kBBytes = kBRows * kDi * 2;            // 128 KB
constexpr uint32_t kBQuarter = kBBytes / 4;               // 32 KB: 256 rows x 64 dims
constexpr int kTmemCols = 512;

struct __align__(1024) PrefillSmem {
  uint8_t b[kBBytes];                 // Q block: [acc half][dim half] of 256 x 64 bf16, swizzled
  uint8_t a[kStages][kATileBytes];    // key tiles: [dim half] of 128 x 64 bf16, swizzled
  float w[kRowsPerBlock][kHi];
  int32_t pos[kRowsPerBlock];
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], qfull;
  uint32_t tmem_base;
  int abort_flag;
};

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major, M=128, N=256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t acc) {
  umma_f16(tmem_d, adesc, bdesc, kIdesc, acc);
}
struct PrefillParams {
  const float* w;
  const int32_t* pos;
  float* scores;
  int64_t ld;
  int64_t max_len;
  int n_rows;
  int n_init, n_loc;
  int tiles_per_cta;   // key tiles per CTA (grid.x splits the key range)
  int* err;
};

__global__ void __launch_bounds__(kThreads, 1)
    index_prefill_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_q,
                         PrefillParams prm) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // The swizzled operand tiles need 1024-byte aligned bases; the dynamic
  // shared-memory window starts on such a boundary. Checked, never assumed.
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) flag_error(prm.err, LSA_DEVERR_TIMEOUT);
    return;
  }
  PrefillSmem& sm = *reinterpret_cast<PrefillSmem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  // Heaviest (latest, longest-context) row blocks first.
  const int blk = gridDim.y - 1 - blockIdx.y;
  const int row0 = blk * kRowsPerBlock;

  if (threadIdx.x < kRowsPerBlock) {
    const int r = row0 + threadIdx.x;
    sm.pos[threadIdx.x] = r < prm.n_rows ? prm.pos[r] : -1;
  }
  for (int i = threadIdx.x; i < kRowsPerBlock * kHi; i += kThreads) {
    const int r = row0 + i / kHi;
    sm.w[i / kHi][i % kHi] = r < prm.n_rows ? prm.w[(int64_t)r * kHi + i % kHi] : 0.f;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.tfull[b], 1);
      mbar_init(&sm.tempty[b], kEpiWarps);
    }
    mbar_init(&sm.qfull, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
  }
  __syncthreads();

  // Key range of this CTA: tiles [t0, t1) clipped to what the block's rows see.
  int pmax = -1;
#pragma unroll
  for (int i = 0; i < kRowsPerBlock; ++i) pmax = max(pmax, sm.pos[i]);
  if (threadIdx.x == 0 && blockIdx.x == 0 && (int64_t)pmax >= prm.max_len) flag_error(prm.err, LSA_DEVERR_POS);
  const int64_t vis = min64((int64_t)pmax + 1, prm.max_len);
  const int n_tiles_blk = (int)((vis + kTileKeys - 1) / kTileKeys);
  const int t0 = blockIdx.x * prm.tiles_per_cta;
  const int t1 = min(n_tiles_blk, t0 + prm.tiles_per_cta);
  if (t0 >= t1) return;  // uniform across the CTA; nothing allocated yet
  const int n_tiles = t1 - t0;

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      mbar_expect_tx(&sm.qfull, kBBytes);
      for (int q = 0; q < 4; ++q)  // [acc half hb][dim half kh] = 256 rows x 64 dims
        tma_load_2d(sm.b + q * kBQuarter, &map_q, (q & 1) * 64, row0 * kHi + (q >> 1) * 256, &sm.qfull);
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&sm.empty[s], ((i / kStages) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&sm.full[s], kATileBytes);
        const int key0 = (t0 + i) * kTileKeys;
        tma_load_2d(sm.a[s], &map_k, 0, key0, &sm.full[s]);
        tma_load_2d(sm.a[s] + kAHalfBytes, &map_k, 64, key0, &sm.full[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool ok = mbar_wait(&sm.qfull, 0, abort_flag);
      const uint32_t b_base = smem_u32(sm.b);
      for (int i = 0; ok && i < n_tiles; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&sm.full[s], (i / kStages) & 1, abort_flag)) break;
        const uint32_t a_base = smem_u32(sm.a[s]);
        for (int hb = 0; hb < 2 && ok; ++hb) {
          // accumulator hb is free once the epilogue drained it for tile i-1
          if (i > 0 && !mbar_wait(&sm.tempty[hb], (i - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + hb * 256;
#pragma unroll
          for (int ks = 0; ks < kDi / 16; ++ks) {
            const int kh = ks >> 2;
            const uint32_t koff = (ks & 3) * 32;
            const uint64_t ad = sw128_desc(a_base + kh * kAHalfBytes + koff);
            const uint64_t bd = sw128_desc(b_base + (hb * 2 + kh) * kBQuarter + koff);
            umma_bf16(d, ad, bd, ks > 0 ? 1u : 0u);
          }
          umma_commit(&sm.tfull[hb]);
        }
        if (!ok) break;
        umma_commit(&sm.empty[s]);  // the stage is free when both halves' MMAs completed
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int e = warp - 2;
    const int quarter = warp & 3;      // tensor-memory lanes this warp may read
    const int tok_half = e >> 2;       // tokens 0-3 or 4-7 within an accumulator
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    for (int i = 0; i < n_tiles; ++i) {
      const int64_t j = (int64_t)(t0 + i) * kTileKeys + quarter * 32 + lane;
      for (int hb = 0; hb < 2; ++hb) {
        // one lane waits, the warp follows its verdict (tcgen05.ld needs the whole warp)
        int ok = 0;
        if (lane == 0) ok = mbar_wait(&sm.tfull[hb], i & 1, abort_flag) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) goto done;
        tc_fence_after();
        // this warp's 4 tokens x 32 heads in one round of loads; the
        // accumulator goes back to the MMA issuer before the math and stores
        float acc[4][32];
        tmem_ld32_x4(tmem + lane_addr + hb * 256 + tok_half * 4 * 32, 32, acc);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tempty[hb]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int tok = hb * 8 + tok_half * 4 + u;
          float s = 0.f;
          const float4* wv = reinterpret_cast<const float4*>(sm.w[tok]);
#pragma unroll
          for (int h4 = 0; h4 < 8; ++h4) {
            const float4 ww = wv[h4];
            s = fmaf(ww.x, fmaxf(acc[u][4 * h4 + 0], 0.f), s);
            s = fmaf(ww.y, fmaxf(acc[u][4 * h4 + 1], 0.f), s);
            s = fmaf(ww.z, fmaxf(acc[u][4 * h4 + 2], 0.f), s);
            s = fmaf(ww.w, fmaxf(acc[u][4 * h4 + 3], 0.f), s);
          }
          const int p = sm.pos[tok];
          if (j <= p && j < prm.max_len) {
            const bool forced = (j < prm.n_init) || (j >= (int64_t)p + 1 - prm.n_loc);
            prm.scores[(int64_t)(row0 + tok) * prm.ld + j] = forced ? INFINITY : s;
          }
        }
      }
    }
  }
done:
  if (*abort_flag && threadIdx.x == 0) flag_error(prm.err, LSA_DEVERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTmemCols));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// 2D bf16 map over [rows, 128] with a box of box_rows x 64 and 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kDi, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kDi * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool index_prefill_supported(const IndexArgs& a) {
  return a.k_off == nullptr && a.n_seq == 1 && a.seq_of_row == nullptr && a.pos_div == 1 && a.n_rows >= kRowsPerBlock &&
         encode_fn() != nullptr;
}

cudaError_t launch_index_prefill(const IndexArgs& a, cudaStream_t st) {
  if (a.n_rows <= 0) return cudaSuccess;
  CUtensorMap map_k, map_q;
  if (!make_map(&map_k, a.k_idx, (uint64_t)a.max_len, kTileKeys)) return cudaErrorInvalidValue;
  if (!make_map(&map_q, a.q_idx, (uint64_t)a.n_rows * kHi, 256)) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = sizeof(PrefillSmem);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(index_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_blocks = (a.n_rows + kRowsPerBlock - 1) / kRowsPerBlock;
  const int64_t max_tiles = (a.max_len + kTileKeys - 1) / kTileKeys;
  // Split the key range when there are too few row blocks to fill the SMs: at
  // least 4 CTAs per SM, at least 32 key tiles per CTA, and among the splits up
  // to 4x that many the one whose CTA count best fills whole waves of one CTA
  // per SM (row blocks that see every key take equal time).
  const int64_t c_max_tiles = max64(1, max_tiles / 32);
  const int64_t c_lo = max64(1, min64((4LL * sms + n_blocks - 1) / n_blocks, c_max_tiles));
  int64_t chunks = c_lo, tiles_per_cta = (max_tiles + c_lo - 1) / c_lo;
  double best = -1.0;
  for (int64_t c = c_lo; c <= min64(4 * c_lo, c_max_tiles); ++c) {
    const int64_t tpc = (max_tiles + c - 1) / c, cc = (max_tiles + tpc - 1) / tpc, n = cc * n_blocks;
    const double eff = (double)n / (double)(((n + sms - 1) / sms) * sms);
    if (eff > best + 1e-9) {
      best = eff;
      chunks = cc;
      tiles_per_cta = tpc;
    }
  }
  PrefillParams p;
  p.w = a.w;
  p.pos = a.pos;
  p.scores = a.scores;
  p.ld = a.ld;
  p.max_len = a.max_len;
  p.n_rows = a.n_rows;
  p.n_init = a.n_init;
  p.n_loc = a.n_loc;
  p.tiles_per_cta = (int)tiles_per_cta;
  p.err = a.err;
  if (n_blocks > 65535) return cudaErrorInvalidValue;
  const cudaError_t e =
      launch_pdl(index_prefill_kernel, dim3((unsigned)chunks, (unsigned)n_blocks), dim3(kThreads), smem, st, map_k,
                 map_q, p);
  count_launches(1);
  return e;
}

}  // namespace lsa
