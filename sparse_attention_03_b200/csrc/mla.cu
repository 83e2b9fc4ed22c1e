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
// Design. One CTA handles one (query row, split of its key list, sub-block):
// eight math warps and one producer warp. The producer gathers each selected
// 1152-byte latent row with one bulk asynchronous copy per lane (the TMA engine
// moves the bytes; no register staging) into a four-stage ring of 32-key tiles
// (rows padded to 1168 bytes so ldmatrix is conflict-free); full/empty
// mbarriers hand stages between producer and math warps, so three tiles are in
// flight while one is computed. S = Q K^T runs on mma.m16n8k16 with the
// 576-dim contraction split four ways across warps: each warp keeps its quarter
// of Q in registers for the whole CTA, and the partial logits are summed through
// shared memory. The online softmax is base-2 and max-subtracted. O += P V runs
// with the 512 value dims split across the warps (64 each, fp32 accumulators in
// registers). A row's key list is cut into splits of whole tiles, balanced per
// row; with more than one split the CTA writes an unnormalised partial
// (O, m, l) and one merge kernel combines the splits of every row and
// sub-block; with one split it writes bf16 output and lse directly. The
// sub-blocks that share a selection (or the MTP draft steps that share one)
// are the grid's third dimension, so one attention launch and at most one
// merge launch cover them all. Gathered indices are bounds-checked against the
// row's visible keys; every wait is bounded.
#include "common.cuh"
#include "kernels.h"
#include "launch.h"
#include "mla_common.cuh"
#include "tc.cuh"

namespace lsa {
namespace {

constexpr int kTK = 32;             // keys per tile
constexpr int kStages = 4;          // tiles in the ring
constexpr int kSRow = kDLat + 8;    // shared row stride (bf16): 1168 bytes
constexpr int kPRow = kTK + 8;      // P row stride (bf16): 80 bytes
constexpr int kMathWarps = 8;
constexpr int kMathThreads = kMathWarps * 32;
constexpr int kThreads = kMathThreads + 32;  // + the producer warp
constexpr int kMaxSplits = 32;
constexpr int kRowBytes = kDLat * 2;  // 1152
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

constexpr int kPartRow = kTK + 8;   // fp32 row stride of the partial logits (conflict-free float2 stores)

struct __align__(128) MlaSmem {
  uint16_t k[kStages][kTK * kSRow];
  // Q rows at start; afterwards the per-warp partial logits
  // [4 dim quarters][2 head halves][16 heads][kPartRow] fp32.
  uint16_t q[kH * kSRow];
  uint16_t p[kH * kPRow];
  float red_max[4][kH];
  float red_sum[4][kH];
  float alpha[kH];
  float fin_m[kH];
  float fin_l[kH];
  int32_t keys[kStages][kTK];  // gathered key of each tile slot, -1 when masked
  int32_t list[kMaxTopk];      // this split's validated keys
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t qbar;
  int abort_flag;
};
static_assert(4 * 2 * 16 * kPartRow * 4 <= kH * kSRow * 2, "partial logits fit in the Q area");
static_assert((kSRow * 2) % 16 == 0 && kRowBytes % 16 == 0, "bulk copies need 16-byte rows");

struct Split {
  int n_split;
  int list_tiles;  // tiles of the longest key list (the split boundaries)
};

__device__ __forceinline__ void bulk_row(void* dst, const void* src, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(kRowBytes), "r"(smem_u32(bar))
      : "memory");
}

// A wait that ignores the abort flag, used once at exit so that no copy is
// still in flight into this CTA's shared memory when it retires.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity))
    if (global_ns() - t0 > kWaitLimitNs) return;
}

// Named barriers: 1 = the eight math warps, 2 + h = the four warps of head half h.
__device__ __forceinline__ void math_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(kMathThreads) : "memory"); }
__device__ __forceinline__ void half_sync(int h) { asm volatile("bar.sync %0, 128;\n" ::"r"(2 + h) : "memory"); }
// Barrier 4 staggers the halves once: half 0 arrives after its first logits,
// half 1 waits for that before starting.
__device__ __forceinline__ void stagger_arrive() { asm volatile("bar.arrive 4, %0;\n" ::"n"(kMathThreads) : "memory"); }
__device__ __forceinline__ void stagger_wait() { asm volatile("bar.sync 4, %0;\n" ::"n"(kMathThreads) : "memory"); }


// Warp roles (math warps 0..7): head half mt = w >> 2 (heads 16mt .. 16mt+15)
// and quarter kq = w & 3, so each SM sub-partition runs one warp of each half
// and the two halves, which share nothing but the key tiles, drift apart and
// overlap one half's softmax with the other's MMAs. Logits: warp w contracts
// dim quarter kq (9 k16 steps) for its 16 heads x 32 keys, Q fragments in
// registers, two accumulator chains per 8-key n-tile; the four quarters meet in
// shared memory. Softmax: warp w owns key group kq (8 keys); each lane one head
// and 4 keys. O += P V: warp w owns value dims 128kq .. 128kq+127 of its heads.
__global__ void __launch_bounds__(kThreads, 1) mla_kernel(MlaArgs a, Split sp, float* part_o,
                                                          float2* part_ml) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  MlaSmem& sm = *reinterpret_cast<MlaSmem*>(smem_raw);
  const int s = blockIdx.x, r = blockIdx.y, z = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.full[i], 32);
      mbar_init(&sm.empty[i], kMathWarps);
    }
    mbar_init(&sm.qbar, 32);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;
  // Forced-first lists: the forced columns are gathered and attended over before
  // the wait for the previous kernel (the top-k that writes idx / count); only
  // the producer's index loads and the epilogue's stores come after it.
  const bool ff = a.forced_first && a.idx;
  if (!ff) pdl_wait();

  // This split's slots: whole tiles of the longest list, clipped to the row's own.
  const int64_t t_lo = (int64_t)sp.list_tiles * s / sp.n_split;
  const int64_t t_hi = (int64_t)sp.list_tiles * (s + 1) / sp.n_split;
  const int64_t b0 = t_lo * kTK;
  const int cap = (int)((t_hi - t_lo) * kTK);

  if (warp == kMathWarps && ff) {
    // ================= producer warp, forced-first list =================
    const uint16_t* __restrict__ qg = a.q[z] + ((int64_t)r * kH + lane) * kDLat;
    mbar_expect_tx(&sm.qbar, kRowBytes);
    bulk_row(&sm.q[lane * kSRow], qg, &sm.qbar);
    const RowGeom geo = row_base(a, r, false);
    const ListPlan lp = list_plan(a, geo.nvis, mtp_ext(a, geo, z, false));
    const FfTiles ft = ff_tiles<kTK>(lp, s, sp.n_split);
    const uint16_t* __restrict__ latb = a.lat[z] + geo.kbase * kDLat;
    int issued = 0;  // tiles handed to the ring (all of them unless the test hook stops early)
    auto issue = [&](int tt, int key) {
      if (tt == a.drop_tile) return false;
      const int i = tt % kStages;
      if (tt >= kStages) mbar_wait(&sm.empty[i], ((tt / kStages) - 1) & 1, abort_flag, a.wait_ns);
      sm.keys[i][lane] = key;
      uint16_t* dst = &sm.k[i][lane * kSRow];
      if (key >= 0) {
        mbar_expect_tx(&sm.full[i], kRowBytes);
        bulk_row(dst, latb + (int64_t)key * kDLat, &sm.full[i]);
      } else {
#pragma unroll 8
        for (int c = 0; c < kDLat / 8; ++c) *reinterpret_cast<uint4*>(dst + 8 * c) = make_uint4(0, 0, 0, 0);
        fence_proxy_async();
        mbar_arrive(&sm.full[i]);
      }
      ++issued;
      return true;
    };
    // the known slots (forced columns, or a dense row's whole list, then any
    // MTP extra keys): keys by formula
    bool go = true;
    for (int tt = 0; go && tt < ft.kt; ++tt)
      go = issue(tt, known_slot_key<kTK>(lp, ft, a, (int64_t)(ft.kt0 + tt) * kTK + lane));
    // the selected slots: the top-k's list, after it has finished
    pdl_wait();
    int c = a.count[r];
    if (c != (int)lp.L && geo.nvis > 0) flag_error(a.err, LSA_DEVERR_COUNT);
    const int64_t uend = max64(lp.K, min64((int64_t)c, lp.L));
    const int32_t* __restrict__ irow = a.idx + (int64_t)r * a.topk;
    constexpr int kBatch = 8;  // tiles whose indices are requested together
    for (int u0 = 0; go && u0 < ft.ut; u0 += kBatch) {
      int key[kBatch];
      bool listed[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int64_t sl = ft.ub + (int64_t)(ft.ut0 + u0 + j) * kTK + lane;
        listed[j] = u0 + j < ft.ut && sl < uend;
        key[j] = listed[j] ? __ldg(irow + sl) : -1;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        if (listed[j] && (key[j] < 0 || key[j] >= geo.nvis)) {
          flag_error(a.err, LSA_DEVERR_INDEX);
          key[j] = -1;
        }
        if (go && u0 + j < ft.ut) go = issue(ft.kt + u0 + j, key[j]);
      }
    }
    // Retire only after every copy into this CTA's shared memory has landed.
    if (lane == 0) {
      mbar_drain(&sm.qbar, 0);
      for (int i = 0; i < kStages && i < issued; ++i) {
        const int last = i + ((issued - 1 - i) / kStages) * kStages;
        mbar_drain(&sm.full[i], (last / kStages) & 1);
      }
    }
    return;
  }

  if (warp == kMathWarps) {
    // ================= producer warp =================
    // Q and the first indices go out before the row geometry is known.
    const uint16_t* __restrict__ qg = a.q[z] + ((int64_t)r * kH + lane) * kDLat;
    mbar_expect_tx(&sm.qbar, kRowBytes);
    bulk_row(&sm.q[lane * kSRow], qg, &sm.qbar);
    const int32_t* __restrict__ irow = a.idx ? a.idx + (int64_t)r * a.topk + b0 : nullptr;
    constexpr int kChunk = 16;
    int v[kChunk];
    // never past this row's topk entries (the tiles round topk up to 32)
    const int first = irow ? (int)min64(min64((int64_t)cap, (int64_t)a.topk - b0), 32 * kChunk) : 0;
#pragma unroll
    for (int u = 0; u < kChunk; ++u) {
      const int i = u * 32 + lane;
      v[u] = (irow && i < first) ? __ldg(irow + i) : 0;
    }
    const RowGeom geo = row_geometry(a, r, false);
    const int nk = (int)max64(0, min64((int64_t)cap, geo.n_list - b0));
    // With an index list the split holds at most topk <= kMaxTopk keys (the
    // launcher sizes the splits from topk); a dense row's keys are b0 + slot, a
    // LoZA row's follow from its position (loza_key): neither needs a list.
    for (int c0 = 0; irow && c0 < nk; c0 += 32 * kChunk) {
      if (c0 > 0) {
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
          const int i = c0 + u * 32 + lane;
          v[u] = (irow && i < nk) ? __ldg(irow + i) : 0;
        }
      }
#pragma unroll
      for (int u = 0; u < kChunk; ++u) {
        const int i = c0 + u * 32 + lane;
        if (i < nk) {
          int64_t key = v[u];
          if (key < 0 || key >= geo.nvis) {
            flag_error(a.err, LSA_DEVERR_INDEX);
            key = -1;
          }
          sm.list[i] = (int32_t)key;
        }
      }
    }
    __syncwarp();
    const int n_tiles = (nk + kTK - 1) / kTK;
    const uint16_t* __restrict__ latb = a.lat[z] + geo.kbase * kDLat;
    const LozaSpan zs = a.loza ? loza_span(a, geo.nvis) : LozaSpan{0, 0};
    // tiles handed to the ring: all of them unless the test hook stops early
    const int issued = a.drop_tile >= 0 ? min(n_tiles, a.drop_tile) : n_tiles;
    for (int base = 0; base < issued; base += kStages) {
#pragma unroll
      for (int i = 0; i < kStages; ++i) {
        const int tt = base + i;
        if (tt < issued) {
          const int sl = tt * kTK + lane;
          const int key = sl >= nk ? -1 : irow ? sm.list[sl] : (int)(a.loza ? loza_key(zs, b0 + sl) : b0 + sl);
          if (tt >= kStages) mbar_wait(&sm.empty[i], ((tt / kStages) - 1) & 1, abort_flag, a.wait_ns);
          sm.keys[i][lane] = key;
          uint16_t* dst = &sm.k[i][lane * kSRow];
          if (key >= 0) {
            mbar_expect_tx(&sm.full[i], kRowBytes);
            bulk_row(dst, latb + (int64_t)key * kDLat, &sm.full[i]);
          } else {
            // a masked slot: zero row (its weight is exactly 0, and 0 * 0 stays finite)
#pragma unroll 8
            for (int c = 0; c < kDLat / 8; ++c) *reinterpret_cast<uint4*>(dst + 8 * c) = make_uint4(0, 0, 0, 0);
            fence_proxy_async();
            mbar_arrive(&sm.full[i]);
          }
        }
      }
    }
    // Retire only after every copy into this CTA's shared memory has landed.
    if (lane == 0) {
      mbar_drain(&sm.qbar, 0);
      for (int i = 0; i < kStages && i < issued; ++i) {
        const int last = i + ((issued - 1 - i) / kStages) * kStages;
        mbar_drain(&sm.full[i], (last / kStages) & 1);
      }
    }
    return;
  }

  // ================= math warps =================
  int n_tiles;
  if (ff) {
    const RowGeom geo = row_base(a, r, s == 0 && tid == 0);
    const FfTiles ft = ff_tiles<kTK>(list_plan(a, geo.nvis, mtp_ext(a, geo, z, s == 0 && tid == 0)), s, sp.n_split);
    n_tiles = ft.kt + ft.ut;
  } else {
    const RowGeom geo = row_geometry(a, r, s == 0 && tid == 0);
    const int nk = (int)max64(0, min64((int64_t)cap, geo.n_list - b0));
    n_tiles = (nk + kTK - 1) / kTK;
  }
  const int g = lane >> 2, t = lane & 3;
  const int mt = warp >> 2, kq = warp & 3;
  mbar_wait(&sm.qbar, 0, abort_flag, a.wait_ns);
  // Q fragments of this warp: heads 16mt .. 16mt+15, k16 steps 9kq .. 9kq+8.
  uint32_t qf[9][4];
  {
    const uint32_t qa = smem_u32(&sm.q[(16 * mt + (lane & 15)) * kSRow + 8 * (lane >> 4)]) + 9 * kq * 32;
#pragma unroll
    for (int ks = 0; ks < 9; ++ks) ldsm_x4(qa + ks * 32, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }
  math_sync();  // every warp holds its Q fragments: the Q area becomes the partial logits
  float* part = reinterpret_cast<float*>(sm.q);

  const float scale_log2 = a.scale * kLog2e;
  // softmax state for this lane's head
  const int sh = 16 * mt + (lane >> 1);
  const int kb4 = 8 * kq + 4 * (lane & 1);
  float m_run = -INFINITY, l_run = 0.f;
  // value accumulators: o[nt][4], heads 16mt+g (+8), dims 128kq + 8nt + 2t
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt)
#pragma unroll
    for (int j = 0; j < 4; ++j) o[nt][j] = 0.f;

  // Half 1 starts one logits phase behind half 0, so that from then on one
  // half's softmax runs while the other issues MMAs (both halves see the same
  // n_tiles, so the barrier is taken by both or by neither).
  if (mt == 1 && n_tiles > 0) stagger_wait();
  for (int tt = 0; tt < n_tiles; ++tt) {
    const int st = tt % kStages;
    mbar_wait(&sm.full[st], (tt / kStages) & 1, abort_flag, a.wait_ns);
    const uint16_t* kt = sm.k[st];

    // ---- partial logits over this warp's dim quarter ----
    float sc[2][4][4];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[c][nt][j] = 0.f;
    const uint32_t kb0 = smem_u32(&kt[((lane & 7) + 8 * (lane >> 4)) * kSRow + 8 * ((lane >> 3) & 1)]) +
                         9 * kq * 32;
#pragma unroll
    for (int ks = 0; ks < 9; ++ks) {
      const int c = ks & 1;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint32_t b[4];
        ldsm_x4(kb0 + (16 * j * kSRow) * 2 + ks * 32, b[0], b[1], b[2], b[3]);
        mma_16816(sc[c][2 * j], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b[0], b[1]);
        mma_16816(sc[c][2 * j + 1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], b[2], b[3]);
      }
    }
    {
      float* pw = part + ((kq * 2 + mt) * 16) * kPartRow;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        *reinterpret_cast<float2*>(&pw[g * kPartRow + 8 * nt + 2 * t]) =
            make_float2(sc[0][nt][0] + sc[1][nt][0], sc[0][nt][1] + sc[1][nt][1]);
        *reinterpret_cast<float2*>(&pw[(g + 8) * kPartRow + 8 * nt + 2 * t]) =
            make_float2(sc[0][nt][2] + sc[1][nt][2], sc[0][nt][3] + sc[1][nt][3]);
      }
    }
    if (mt == 0 && tt == 0) stagger_arrive();
    half_sync(mt);  // (1) this half's partials complete

    // ---- sum the partials, mask, tile max (lane: head sh, keys kb4 .. kb4+3) ----
    float x[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      const float4 vv =
          *reinterpret_cast<const float4*>(part + ((q4 * 2 + mt) * 16 + (lane >> 1)) * kPartRow + kb4);
      x[0] += vv.x; x[1] += vv.y; x[2] += vv.z; x[3] += vv.w;
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[i] = sm.keys[st][kb4 + i] >= 0 ? x[i] * scale_log2 : -INFINITY;
      mx = fmaxf(mx, x[i]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    if ((lane & 1) == 0) sm.red_max[kq][sh] = mx;
    half_sync(mt);  // (2) tile maxima
    const float tmax = fmaxf(fmaxf(sm.red_max[0][sh], sm.red_max[1][sh]), fmaxf(sm.red_max[2][sh], sm.red_max[3][sh]));
    const float m_new = fmaxf(m_run, tmax);
    const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = exp2f(m_run - m_use);
    m_run = m_new;
    const float p0 = exp2f(x[0] - m_use), p1 = exp2f(x[1] - m_use);
    const float p2 = exp2f(x[2] - m_use), p3 = exp2f(x[3] - m_use);
    float ps = (p0 + p1) + (p2 + p3);
    *reinterpret_cast<uint2*>(&sm.p[sh * kPRow + kb4]) = make_uint2(pack_bf16x2(p0, p1), pack_bf16x2(p2, p3));
    ps += __shfl_xor_sync(0xffffffffu, ps, 1);
    if ((lane & 1) == 0) {
      sm.red_sum[kq][sh] = ps;
      if (kq == 0) sm.alpha[sh] = alpha;
    }
    half_sync(mt);  // (3) P, alpha and tile sums of this half ready
    l_run = l_run * alpha +
            ((sm.red_sum[0][sh] + sm.red_sum[1][sh]) + (sm.red_sum[2][sh] + sm.red_sum[3][sh]));

    // ---- O += P V, heads of this half, value dims 128kq .. 128kq+127 ----
    {
      const float al0 = sm.alpha[16 * mt + g], al1 = sm.alpha[16 * mt + 8 + g];
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        o[nt][0] *= al0;
        o[nt][1] *= al0;
        o[nt][2] *= al1;
        o[nt][3] *= al1;
      }
    }
    const uint32_t pa = smem_u32(&sm.p[(16 * mt + (lane & 15)) * kPRow + 8 * (lane >> 4)]);
    const uint32_t vb0 =
        smem_u32(&kt[((lane & 7) + 8 * ((lane >> 3) & 1)) * kSRow + 128 * kq + 8 * (lane >> 4)]);
#pragma unroll
    for (int kk = 0; kk < kTK / 16; ++kk) {
      uint32_t pf[4];
      ldsm_x4(pa + kk * 32, pf[0], pf[1], pf[2], pf[3]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t vv[4];
        ldsm_x4_t(vb0 + (kk * 16 * kSRow + 16 * np) * 2, vv[0], vv[1], vv[2], vv[3]);
        mma_16816(o[2 * np], pf[0], pf[1], pf[2], pf[3], vv[0], vv[1]);
        mma_16816(o[2 * np + 1], pf[0], pf[1], pf[2], pf[3], vv[2], vv[3]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);  // this warp is done with the stage
  }
  pdl_trigger();
  if (kq == 0 && (lane & 1) == 0) {
    sm.fin_m[sh] = m_run;
    sm.fin_l[sh] = l_run;
  }
  math_sync();
  if (tid == 0 && *abort_flag) flag_error(a.err, LSA_DEVERR_TIMEOUT);

  // ---- epilogue ----
  if (ff) pdl_wait();  // the outputs and the split-K workspace may still be read by earlier kernels
  const int h0 = 16 * mt + g, h1 = h0 + 8;
  if (sp.n_split == 1) {
    uint16_t* __restrict__ og = a.out[z] + (int64_t)r * kH * kDV;
    const float l0 = sm.fin_l[h0], l1 = sm.fin_l[h1];
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 128 * kq + 8 * nt + 2 * t;
      *reinterpret_cast<uint32_t*>(&og[h0 * kDV + d]) = pack_bf16x2(o[nt][0] * i0, o[nt][1] * i0);
      *reinterpret_cast<uint32_t*>(&og[h1 * kDV + d]) = pack_bf16x2(o[nt][2] * i1, o[nt][3] * i1);
    }
    if (a.lse[z] && tid < kH) {
      const float l = sm.fin_l[tid];
      a.lse[z][(int64_t)r * kH + tid] = l > 0.f ? (sm.fin_m[tid] + log2f(l)) * kLn2 : -INFINITY;
    }
  } else {
    const int64_t base = ((int64_t)z * a.n_rows + r) * sp.n_split + s;
    float* __restrict__ po = part_o + base * kH * kDV;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 128 * kq + 8 * nt + 2 * t;
      *reinterpret_cast<float2*>(&po[h0 * kDV + d]) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(&po[h1 * kDV + d]) = make_float2(o[nt][2], o[nt][3]);
    }
    if (tid < kH) part_ml[base * kH + tid] = make_float2(sm.fin_m[tid], sm.fin_l[tid]);
  }
}

// One CTA per (head, row, sub-block): 128 threads x 4 value dims, so that a
// small decode batch still spreads the merge over many SMs. Every thread issues
// its partial-output loads before the split weights are known, so the two
// reads overlap.
__global__ void __launch_bounds__(128) mla_merge_kernel(MlaArgs a, Split sp, const float* part_o,
                                                        const float2* part_ml) {
  __shared__ float wgt[kMaxSplits];
  __shared__ float inv_l;
  pdl_wait();
  pdl_trigger();  // the next MLA may start its forced columns; it waits for this grid before writing
  const int h = blockIdx.x, r = blockIdx.y, z = blockIdx.z, tid = threadIdx.x;
  const int64_t base = ((int64_t)z * a.n_rows + r) * sp.n_split;
  const int e = tid * 4;
  constexpr int kIn = 8;  // partial rows in flight per thread
  float4 v[kIn];
#pragma unroll
  for (int i = 0; i < kIn; ++i)
    v[i] = i < sp.n_split ? *reinterpret_cast<const float4*>(part_o + ((base + i) * kH + h) * kDV + e)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid < 32) {
    const float2 ml = tid < sp.n_split ? part_ml[(base + tid) * kH + h] : make_float2(-INFINITY, 0.f);
    float M = ml.x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float wv = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
    float L = wv * ml.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (tid < sp.n_split) wgt[tid] = wv;
    if (tid == 0) {
      inv_l = L > 0.f ? 1.f / L : 0.f;
      if (a.lse[z]) a.lse[z][(int64_t)r * kH + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
    }
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto add = [&](const float4& x, float wv) {
    acc.x = fmaf(wv, x.x, acc.x);
    acc.y = fmaf(wv, x.y, acc.y);
    acc.z = fmaf(wv, x.z, acc.z);
    acc.w = fmaf(wv, x.w, acc.w);
  };
#pragma unroll
  for (int i = 0; i < kIn; ++i)
    if (i < sp.n_split) add(v[i], wgt[i]);
  for (int s = kIn; s < sp.n_split; ++s)
    add(*reinterpret_cast<const float4*>(part_o + ((base + s) * kH + h) * kDV + e), wgt[s]);
  const float il = inv_l;
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * il, acc.y * il);
  pk.y = pack_bf16x2(acc.z * il, acc.w * il);
  *reinterpret_cast<uint2*>(a.out[z] + ((int64_t)r * kH + h) * kDV + e) = pk;
}

}  // namespace

size_t mla_ws_bytes(int n_rows, int n_sub, int n_split) {
  if (n_split <= 1) return 0;
  const size_t per = (size_t)kH * kDV * sizeof(float) + (size_t)kH * sizeof(float2);
  return (size_t)n_rows * n_sub * n_split * per + 256;
}

int mla_choose_splits(int n_rows, int n_sub, int64_t max_list, bool forced_first) {
  // One wave at one CTA per SM: split the rows' key lists until the CTAs cover
  // the SMs, keeping at least four tiles per split (the ring's depth) and at
  // most kMaxSplits splits. With forced-first lists the CTAs start while the
  // top-k is still finishing, which holds one SM per row (its last CTA): leave
  // those SMs out, so that no CTA starts only after the top-k, unless that
  // would leave more SMs idle than the late CTAs cost (at most an eighth of
  // the CTAs start late).
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t work = max64((int64_t)n_rows * n_sub, 1);
  int64_t per = sms / work;
  if (forced_first) {
    const int64_t free_sms = max(sms - n_rows, sms / 2);
    const int64_t reserved = free_sms / work;
    if (per > reserved && per * work - free_sms > per * work / 8) per = reserved;
  }
  const int64_t by_len = (max_list + kStages * kTK - 1) / (kStages * kTK);
  int64_t n = min64(by_len, per);
  n = max64(1, min64(n, kMaxSplits));
  return (int)n;
}

namespace {
thread_local long long t_test_wait_ns = 0;
thread_local int t_test_drop = -1;
}  // namespace

void mla_arm_wait_test(long long wait_ns, int drop_tile) {
  t_test_wait_ns = wait_ns;
  t_test_drop = drop_tile;
}

cudaError_t launch_mla(const MlaArgs& a_in, cudaStream_t st) {
  if (a_in.n_rows <= 0) return cudaSuccess;
  MlaArgs a = a_in;
  if (t_test_drop >= 0 || t_test_wait_ns > 0) {  // the armed test hook applies to this launch only
    a.drop_tile = t_test_drop;
    if (t_test_wait_ns > 0) a.wait_ns = t_test_wait_ns;
    t_test_drop = -1;
    t_test_wait_ns = 0;
  }
  int n_split = mla_choose_splits(a.n_rows, a.n_sub, a.max_list, a.forced_first && a.idx);
  // Shrink split-K to what the workspace holds.
  while (n_split > 1 && mla_ws_bytes(a.n_rows, a.n_sub, n_split) > a.ws_bytes) --n_split;
  Split sp;
  sp.n_split = n_split;
  // With an index list no row has more than topk keys (the shared list's size).
  const int64_t max_list = a.idx ? min64(a.max_list, (int64_t)min(a.topk, kMaxTopk)) : a.max_list;
  sp.list_tiles = (int)((max_list + kTK - 1) / kTK);
  float* part_o = nullptr;
  float2* part_ml = nullptr;
  if (n_split > 1) {
    uintptr_t p = (reinterpret_cast<uintptr_t>(a.ws) + 255) & ~uintptr_t(255);
    part_o = reinterpret_cast<float*>(p);
    part_ml = reinterpret_cast<float2*>(part_o + (size_t)a.n_rows * a.n_sub * n_split * kH * kDV);
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
      for (int z = 0; z < a.n_sub; ++z) {
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
    cudaError_t e = launch_pdl(mla_kernel, dim3(n_split, nr, a.n_sub), dim3(kThreads), sizeof(MlaSmem), st, b,
                               sp, part_o, part_ml);
    if (e != cudaSuccess) return e;
    if (n_split > 1) {
      e = launch_pdl(mla_merge_kernel, dim3(kH, nr, a.n_sub), dim3(128), 0, st, b, sp, (const float*)part_o,
                     (const float2*)part_ml);
      if (e != cudaSuccess) return e;
    }
    count_launches(n_split > 1 ? 2 : 1);
  }
  return cudaSuccess;
}

}  // namespace lsa
