// The indexer's own projections and the key-cache append (upstream of the
// scored path).
//
// [Lite-Sparse] "LSA（LongCat 稀疏注意力）" (the indexer's structure): wq_b maps
// the q-LoRA representation to 32 heads x 128 dims, wk maps the hidden state to
// the index key, which is RMS-normalised, weights_proj gives one scalar per
// index head, and the index query and key share MLA's RoPE configuration
// (qk_rope_head_dim 64, rope_theta).
// Readings: RoPE on the last 64 of the 128 dims in rotate-half form (pairs
// (i, i + 32), angle pos * theta^(-2i/64)), no rope scaling; RMSNorm with eps
// 1e-6 and a per-dim weight; no scale on the head weights.
//
// Design. Three skinny GEMMs out = X W^T (X [rows, K] bf16, W [N, K] bf16, fp32
// accumulate and fp32 out into the workspace) on mma.m16n8k16: 64 x 64 output
// tiles, K in steps of 32 through a double-buffered cp.async tile with padded
// rows (conflict-free ldmatrix). At decode the rows are few and the kernel
// streams the weights once; at prefill they stay in L2. Then one CTA per row
// normalises the key, rotates the rope dims of the key and of all 32 query heads
// (angles formed and reduced in fp64: positions reach ~10^6), writes the bf16
// query, the fp32 head weights and the bf16 key row into the cache at the row's
// position.
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "launch.h"

namespace lsa {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 32;
constexpr int kGemmThreads = 128;
constexpr int kPad = kBK + 8;  // 80-byte rows: ldmatrix rows fall in distinct bank groups

struct __align__(16) GemmSmem {
  uint16_t a[2][kBM * kPad];
  uint16_t b[2][kBN * kPad];
};

// out[M, N] (row stride N) = X[M, K] (row stride K) . W[N, K]^T; K % 32 == 0.
// With split_k > 1, CTA z covers a slice of K and adds its partial product into
// out (zeroed by the caller): few rows (decode) still give every SM weight
// bytes in flight.
__global__ void __launch_bounds__(kGemmThreads) gemm_tn_kernel(const uint16_t* __restrict__ x,
                                                               const uint16_t* __restrict__ w, float* __restrict__ out,
                                                               int M, int N, int K, int split_k) {
  __shared__ GemmSmem sm;
  pdl_wait();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = blockIdx.x * kBN, m0 = blockIdx.y * kBM;
  // stage loader: 64 rows x 64 B for A and for B, 2 chunks of 16 B per thread each
  auto load = [&](int kt, int st) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int c = tid + kGemmThreads * u;  // 0..255
      const int row = c >> 2, col = (c & 3) * 8;
      const int ma = m0 + row, nb = n0 + row;
      cp_async16(smem_u32(&sm.a[st][row * kPad + col]), ma < M ? x + (int64_t)ma * K + kt * kBK + col : x,
                 ma < M ? 16 : 0);
      cp_async16(smem_u32(&sm.b[st][row * kPad + col]), nb < N ? w + (int64_t)nb * K + kt * kBK + col : w,
                 nb < N ? 16 : 0);
    }
  };
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const int all_kt = K / kBK;
  const int kt0 = (int)((int64_t)all_kt * blockIdx.z / split_k);
  const int n_kt = (int)((int64_t)all_kt * (blockIdx.z + 1) / split_k) - kt0;
  if (n_kt > 0) load(kt0, 0);
  cp_async_commit();
  for (int kt = 0; kt < n_kt; ++kt) {
    const int st = kt & 1;
    if (kt + 1 < n_kt) load(kt0 + kt + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < kBK / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(smem_u32(&sm.a[st][(16 * warp + (lane & 15)) * kPad + 16 * ks + 8 * (lane >> 4)]), a0, a1, a2, a3);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t b[4];
        ldsm_x4(smem_u32(&sm.b[st][(16 * j + (lane & 7) + 8 * (lane >> 4)) * kPad + 16 * ks + 8 * ((lane >> 3) & 1)]),
                b[0], b[1], b[2], b[3]);
        mma_16816(acc[2 * j], a0, a1, a2, a3, b[0], b[1]);
        mma_16816(acc[2 * j + 1], a0, a1, a2, a3, b[2], b[3]);
      }
    }
    __syncthreads();  // the stage is rewritten two iterations on
  }
  pdl_trigger();
  // acc[nt][0..1]: row 16w+g, cols 8nt+2t (+1); acc[nt][2..3]: row 16w+g+8
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const int col = n0 + 8 * nt + 2 * t;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int row = m0 + 16 * warp + g + 8 * hf;
      if (row < M) {
        float* o = out + (int64_t)row * N + col;
        if (split_k == 1) {
          if (col < N) o[0] = acc[nt][2 * hf];
          if (col + 1 < N) o[1] = acc[nt][2 * hf + 1];
        } else {
          if (col < N) atomicAdd(o, acc[nt][2 * hf]);
          if (col + 1 < N) atomicAdd(o + 1, acc[nt][2 * hf + 1]);
        }
      }
    }
  }
}

struct ProjectArgs {
  const float* q;        // [rows, 32 * 128] fp32 (wq_b c_q)
  const float* k;        // [rows, 128] fp32 (wk h)
  const float* wh;       // [rows, 32] fp32 (weights_proj h)
  const uint16_t* k_norm_w;  // [128] bf16
  const int32_t* seq_of_row;
  const int32_t* pos;
  const int64_t* k_off;
  int n_rows, n_seq;
  int64_t max_len;
  double inv_freq[32];   // theta^(-2i/64)
  uint16_t* q_out;       // [rows, 32, 128] bf16
  float* w_out;          // [rows, 32]
  uint16_t* k_cache;     // packed [sum L, 128] bf16
  int* err;
};

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// cos and sin of the RoPE angle pos * inv_freq (inv_freq = theta^(-2i/64), from the
// host in fp64): the angle is formed and reduced to [-pi, pi] in fp64 (positions
// reach ~10^6 radians, where an fp32 angle would be off by tenths), then the
// fp32 sincos of the reduced angle.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, double inv_freq, float& c, float& s) {
  const double two_pi = 6.283185307179586476925;
  const double ang = (double)pos * inv_freq;
  const double r = fma(-rint(ang * (1.0 / two_pi)), two_pi, ang);
  sincosf((float)r, &s, &c);
}

// One CTA (128 threads, thread = dim d) per row.
__global__ void __launch_bounds__(128) project_epilogue_kernel(ProjectArgs a) {
  __shared__ float kv[kDi];
  __shared__ float red[4];
  pdl_wait();
  const int r = blockIdx.x, d = threadIdx.x, lane = d & 31, warp = d >> 5;
  // the row's cache slot: sequence start + position (clamped and flagged, never written out of range)
  const int seq = a.seq_of_row ? a.seq_of_row[r] : (a.k_off ? r : 0);
  const int64_t p = a.pos[r];
  bool ok = seq >= 0 && seq < a.n_seq && p >= 0 && p < a.max_len;
  int64_t slot = p;
  if (ok && a.k_off) {
    const int64_t base = a.k_off[seq], len = a.k_off[seq + 1] - base;
    ok = p < len;
    slot = base + p;
  }
  if (!ok && d == 0) flag_error(a.err, (seq < 0 || seq >= a.n_seq) ? LSA_DEVERR_SEQ : LSA_DEVERR_POS);
  // RoPE angle of this dim's pair (dims 64..127; pair i = (d - 64) % 32)
  float c = 1.f, s = 0.f;
  const bool rot = d >= kDi - 64;
  if (rot) {
    rope_cos_sin(p, a.inv_freq[(d - (kDi - 64)) & 31], c, s);
  }
  const bool first_half = d < kDi - 32;  // (a, b) pair: a = dim d, b = dim d + 32
  // ---- key: RMSNorm then RoPE ----
  const float kr = a.k[(int64_t)r * kDi + d];
  float ss = kr * kr;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  const float inv = 1.f / sqrtf((red[0] + red[1] + red[2] + red[3]) / kDi + 1e-6f);
  const float kn = kr * inv * bf16_to_f32(a.k_norm_w[d]);
  kv[d] = kn;
  __syncthreads();
  float ko = kn;
  if (rot) ko = first_half ? kn * c - kv[d + 32] * s : kv[d - 32] * s + kn * c;
  if (ok) a.k_cache[slot * kDi + d] = f32_to_bf16_rne(ko);
  // ---- head weights ----
  if (d < kHi) a.w_out[(int64_t)r * kHi + d] = a.wh[(int64_t)r * kHi + d];
  // ---- query: RoPE of every head ----
  const float* __restrict__ qr = a.q + (int64_t)r * kHi * kDi;
  uint16_t* __restrict__ qo = a.q_out + (int64_t)r * kHi * kDi;
#pragma unroll 4
  for (int h = 0; h < kHi; ++h) {
    const float v = qr[h * kDi + d];
    float o = v;
    if (rot) o = first_half ? v * c - qr[h * kDi + d + 32] * s : qr[h * kDi + d - 32] * s + v * c;
    qo[h * kDi + d] = f32_to_bf16_rne(o);
  }
  pdl_trigger();
}

// ---------------------------------------------------------------------------
// Few rows (decode): one launch for all three projections and the epilogue.
//
// The weights (12.6 MB of wq_b, 0.8 MB of wk, 0.2 MB of weights_proj) are the
// only real traffic, so they are spread evenly over one wave of 8-CTA clusters,
// about 96 KB of weights per CTA: 16 clusters take two query heads each (4 CTAs
// per head, each a quarter of q_lora), one cluster takes wk and one
// weights_proj (8 CTAs each, an eighth of the hidden size). 144 CTAs, so the 18
// clusters fit in one wave (at most 33 such clusters are resident at once). A
// warp takes 16 weight rows as the M dimension of mma.m16n8k16 (A fragments
// loaded straight from HBM with 16-byte loads, three 64-wide k-steps in flight)
// and 16 token rows as two n8 tiles (B fragments from the CTA's token slice in
// shared memory); the contraction dimension is permuted the same way on both
// sides, which leaves every dot product unchanged. Each CTA stores its partial
// sums straight into the shared memory of the CTA of its tile that finishes
// those rows (distributed shared memory); after one cluster barrier the owner
// adds the K slices in a fixed order and runs the RMSNorm / RoPE epilogue above
// on its 16 / (CTAs per tile) rows.
constexpr int kSplit = 8;          // CTAs per cluster
constexpr int kQSplit = 4;         // CTAs per query head (K slices of q_lora)
constexpr int kFusedWarps = 8;     // 8 x 16 = 128 output columns per tile
constexpr int kFusedThreads = kFusedWarps * 32;
constexpr int kFusedRows = 16;     // token rows per CTA
constexpr int kQClusters = kHi * kQSplit / kSplit;
constexpr int kFusedClusters = kQClusters + 2;
constexpr int kFusedMaxRows = 64;  // 4 row blocks; more rows take the tiled GEMMs
constexpr int kFusedMaxSlice = 1024;  // K slice; the token slice then takes <= 16 x 2112 bytes of shared memory
constexpr int kMaxPass = kFusedRows / (kFusedThreads / kDi) / kQSplit;  // epilogue rows per thread

struct FusedArgs {
  const uint16_t* c_q;
  const uint16_t* hidden;
  const uint16_t* wq_b;
  const uint16_t* wk;
  const uint16_t* wproj;
  const uint16_t* k_norm_w;
  const int32_t* seq_of_row;
  const int32_t* pos;
  const int64_t* k_off;
  int n_rows, n_seq, q_lora, hidden_dim;
  int64_t max_len;
  double inv_freq[32];  // theta^(-2i/64)
  uint16_t* q_out;
  float* w_out;
  uint16_t* k_cache;
  int* err;
};

struct WFrag {
  uint4 lo[2];  // weight row g:   chunks 4c + t of the 64-wide k-step, c = 0, 1
  uint4 hi[2];  // weight row g+8
};

__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kFusedThreads, 2)
    project_fused_kernel(FusedArgs a) {
  extern __shared__ __align__(16) unsigned char xs[];  // token slice [16][ks * 2 + 64 bytes]
  __shared__ float recv[kFusedRows][kDi];  // [source CTA of the tile x local row][column]
  __shared__ float val[2][kDi];
  __shared__ float red[2][4];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int cl = blockIdx.x / kSplit;
  const int rank = (int)cluster_rank();
  const int r0 = blockIdx.y * kFusedRows;

  // kind 0: wk (128 columns), 1: weights_proj (32), 2: wq_b rows of query head `head`
  const int kind = cl < kQClusters ? 2 : cl - kQClusters;
  const int gsize = kind == 2 ? kQSplit : kSplit;  // CTAs sharing this CTA's tile
  const int grank = rank % gsize, gbase = rank - grank;
  const int head = kind == 2 ? cl * (kSplit / kQSplit) + rank / kQSplit : 0;
  const int K = kind == 2 ? a.q_lora : a.hidden_dim;
  const int ncol = kind == 1 ? kHi : kDi;
  const uint16_t* __restrict__ W = kind == 0 ? a.wk : kind == 1 ? a.wproj : a.wq_b + (int64_t)head * kDi * K;
  const uint16_t* __restrict__ X = kind == 2 ? a.c_q : a.hidden;
  const int ks = K / gsize, k0 = grank * ks, n_steps = ks / 64;
  const int xstride = ks * 2 + 64;  // bytes; == 64 mod 128, so a quarter-warp's two rows use distinct banks
  const int m0 = warp * 16;
  const bool active = m0 < ncol;

  pdl_wait();
  // Weight fragments: a 3-deep register ring of 16-byte loads (chunks of weight
  // rows g and g + 8 at k offsets 0 and 32 of each 64-wide step).
  const uint16_t* __restrict__ w0 = W + (int64_t)(m0 + g) * K + k0 + 8 * t;
  const uint16_t* __restrict__ w1 = w0 + 8LL * K;
  auto load = [&](WFrag& f, int s) {
    if (active && s < n_steps) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        f.lo[c] = ld_stream_v4(w0 + s * 64 + 32 * c);
        f.hi[c] = ld_stream_v4(w1 + s * 64 + 32 * c);
      }
    }
  };
  WFrag f0, f1, f2;
  load(f0, 0);
  load(f1, 1);
  load(f2, 2);
  // token slice -> shared memory (rows past n_rows are zero)
  {
    const int cpr = ks / 8;  // 16-byte chunks per row
    for (int i = tid; i < kFusedRows * cpr; i += kFusedThreads) {
      const int rr = i / cpr, cc = i - rr * cpr;
      const bool in = r0 + rr < a.n_rows;
      cp_async16(smem_u32(xs + rr * xstride + cc * 16), X + (int64_t)(in ? r0 + rr : 0) * K + k0 + cc * 8, in ? 16 : 0);
    }
    cp_async_commit();
  }

  // This CTA's epilogue rows (16 / gsize of them, two at a time): geometry and
  // RoPE cos / sin, while the loads fly.
  const int rsel = tid >> 7, d = tid & (kDi - 1);
  const int rows_per = kFusedRows / gsize, n_pass = rows_per / 2;
  const bool rot = d >= kDi - 64;
  int64_t slot[kMaxPass];
  bool ok[kMaxPass];
  int why[kMaxPass];
  float cs[kMaxPass], sn[kMaxPass];
#pragma unroll
  for (int ps = 0; ps < kMaxPass; ++ps) {
    const int row = r0 + rows_per * grank + 2 * ps + rsel;
    int64_t p = 0;
    slot[ps] = 0;
    ok[ps] = false;
    why[ps] = 0;
    cs[ps] = 1.f;
    sn[ps] = 0.f;
    if (ps < n_pass && row < a.n_rows) {
      if (kind == 0) {
        const int seq = a.seq_of_row ? a.seq_of_row[row] : (a.k_off ? row : 0);
        p = a.pos[row];
        bool good = seq >= 0 && seq < a.n_seq && p >= 0 && p < a.max_len;
        slot[ps] = p;
        if (good && a.k_off) {
          const int64_t base = a.k_off[seq], len = a.k_off[seq + 1] - base;
          good = p < len;
          slot[ps] = base + p;
        }
        ok[ps] = good;
        why[ps] = (seq < 0 || seq >= a.n_seq) ? LSA_DEVERR_SEQ : LSA_DEVERR_POS;
      } else {
        p = a.pos[row];
      }
      if (rot && kind != 1) rope_cos_sin(p, a.inv_freq[(d - (kDi - 64)) & 31], cs[ps], sn[ps]);
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  if (active) {
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    auto step = [&](const WFrag& f, int s) {
      uint4 xb[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c)
          xb[nt][c] = *reinterpret_cast<const uint4*>(xs + (8 * nt + g) * xstride + s * 128 + (4 * c + t) * 16);
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0 = h ? f.lo[c].z : f.lo[c].x, a1 = h ? f.hi[c].z : f.hi[c].x;
          const uint32_t a2 = h ? f.lo[c].w : f.lo[c].y, a3 = h ? f.hi[c].w : f.hi[c].y;
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
            mma_16816(acc[nt], a0, a1, a2, a3, h ? xb[nt][c].z : xb[nt][c].x, h ? xb[nt][c].w : xb[nt][c].y);
        }
    };
    for (int s = 0; s < n_steps; s += 3) {
      step(f0, s);
      load(f0, s + 3);
      if (s + 1 < n_steps) step(f1, s + 1);
      load(f1, s + 4);
      if (s + 2 < n_steps) step(f2, s + 2);
      load(f2, s + 5);
    }
    // acc[nt][e] = (weight row m0+g, token 8nt+2t+e); acc[nt][2+e] = (weight row m0+g+8, same token).
    // Each token row's partials go straight into the shared memory of the CTA
    // that finishes that row, in the slot of this CTA's K slice.
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tr = 8 * nt + 2 * t + e, owner = tr / rows_per, lr = tr - owner * rows_per;
        const uint32_t dst = gbase + owner;
        st_peer_f32(smem_u32(&recv[grank * rows_per + lr][m0 + g]), dst, acc[nt][e]);
        st_peer_f32(smem_u32(&recv[grank * rows_per + lr][m0 + g + 8]), dst, acc[nt][2 + e]);
      }
  }
  pdl_trigger();
  cluster_arrive();  // release: the partials above are visible to their owners after the wait
  cluster_wait();

  // full dot products of this CTA's rows: the tile's K slices summed in order
  float vs[kMaxPass];
#pragma unroll
  for (int ps = 0; ps < kMaxPass; ++ps) {
    vs[ps] = 0.f;
    if (ps < n_pass && d < ncol)
      for (int src = 0; src < gsize; ++src) vs[ps] += recv[src * rows_per + 2 * ps + rsel][d];
  }

#pragma unroll
  for (int ps = 0; ps < kMaxPass; ++ps) {
    if (ps >= n_pass) break;
    const int row = r0 + rows_per * grank + 2 * ps + rsel;
    float v = vs[ps];
    if (kind == 0) {  // key: RMSNorm, then RoPE, into the cache slot
      float ss = v * v;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) red[rsel][warp & 3] = ss;
      __syncthreads();
      const float inv = 1.f / sqrtf((red[rsel][0] + red[rsel][1] + red[rsel][2] + red[rsel][3]) / kDi + 1e-6f);
      v = v * inv * bf16_to_f32(a.k_norm_w[d]);
    }
    if (kind != 1) {
      val[rsel][d] = v;
      __syncthreads();
      if (rot) v = d < kDi - 32 ? v * cs[ps] - val[rsel][d + 32] * sn[ps] : val[rsel][d - 32] * sn[ps] + v * cs[ps];
    }
    if (row < a.n_rows) {
      if (kind == 0) {
        if (ok[ps]) a.k_cache[slot[ps] * kDi + d] = f32_to_bf16_rne(v);
        if (!ok[ps] && d == 0) flag_error(a.err, why[ps]);
      } else if (kind == 1) {
        if (d < kHi) a.w_out[(int64_t)row * kHi + d] = v;
      } else {
        a.q_out[(int64_t)row * kHi * kDi + head * kDi + d] = f32_to_bf16_rne(v);
      }
    }
    __syncthreads();  // val / red are reused by the next pass
  }
}

}  // namespace

size_t project_ws_bytes(int n_rows) { return (size_t)n_rows * (kHi * kDi + kDi + kHi) * sizeof(float) + 256; }

cudaError_t launch_index_project(const ProjectLaunch& L, cudaStream_t st) {
  if (L.n_rows <= 0) return cudaSuccess;
  // Few rows: the single fused launch (K slices of 64-wide steps: q_lora in 4, the hidden size in 8).
  const int ks_max = L.q_lora / kQSplit > L.hidden_dim / kSplit ? L.q_lora / kQSplit : L.hidden_dim / kSplit;
  if (L.n_rows <= kFusedMaxRows && L.q_lora % (kQSplit * 64) == 0 && L.hidden_dim % (kSplit * 64) == 0 &&
      ks_max <= kFusedMaxSlice) {
    FusedArgs f;
    f.c_q = L.c_q;
    f.hidden = L.hidden;
    f.wq_b = L.wq_b;
    f.wk = L.wk;
    f.wproj = L.wproj;
    f.k_norm_w = L.k_norm_w;
    f.seq_of_row = L.seq_of_row;
    f.pos = L.pos;
    f.k_off = L.k_off;
    f.n_rows = L.n_rows;
    f.n_seq = L.n_seq;
    f.q_lora = L.q_lora;
    f.hidden_dim = L.hidden_dim;
    f.max_len = L.max_len;
    for (int i = 0; i < 32; ++i) f.inv_freq[i] = std::pow(L.theta, -2.0 * i / 64.0);
    f.q_out = L.q_out;
    f.w_out = L.w_out;
    f.k_cache = L.k_cache;
    f.err = L.err;
    const size_t smem = (size_t)kFusedRows * (ks_max * 2 + 64);
    const cudaError_t e =
        launch_pdl(project_fused_kernel, dim3(kFusedClusters * kSplit, (L.n_rows + kFusedRows - 1) / kFusedRows),
                   dim3(kFusedThreads), smem, st, f);
    count_launches(1);
    return e;
  }
  float* q = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(L.ws) + 255) & ~uintptr_t(255));
  float* k = q + (size_t)L.n_rows * kHi * kDi;
  float* wh = k + (size_t)L.n_rows * kDi;
  const int my = (L.n_rows + kBM - 1) / kBM;
  if (my > 65535) return cudaErrorInvalidValue;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // split K until the tiles cover the SMs about four times (at least 4 k-steps a slice)
  auto split = [&](int n_tiles, int K) {
    const int64_t want = (4LL * sms + n_tiles - 1) / n_tiles;
    return (int)max64(1, min64(want, K / kBK / 4));
  };
  const int sq = split(my * (kHi * kDi / kBN), L.q_lora), sk = split(my * (kDi / kBN), L.hidden_dim),
            sw = split(my, L.hidden_dim);
  cudaError_t e;
  if (sq > 1 || sk > 1 || sw > 1) {
    e = cudaMemsetAsync(q, 0, (size_t)L.n_rows * (kHi * kDi + kDi + kHi) * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(gemm_tn_kernel, dim3(kHi * kDi / kBN, my, sq), dim3(kGemmThreads), 0, st, L.c_q, L.wq_b, q, L.n_rows,
                 kHi * kDi, L.q_lora, sq);
  if (e != cudaSuccess) return e;
  e = launch_pdl(gemm_tn_kernel, dim3(kDi / kBN, my, sk), dim3(kGemmThreads), 0, st, L.hidden, L.wk, k, L.n_rows, kDi,
                 L.hidden_dim, sk);
  if (e != cudaSuccess) return e;
  e = launch_pdl(gemm_tn_kernel, dim3(1, my, sw), dim3(kGemmThreads), 0, st, L.hidden, L.wproj, wh, L.n_rows, kHi,
                 L.hidden_dim, sw);
  if (e != cudaSuccess) return e;
  ProjectArgs a;
  a.q = q;
  a.k = k;
  a.wh = wh;
  a.k_norm_w = L.k_norm_w;
  a.seq_of_row = L.seq_of_row;
  a.pos = L.pos;
  a.k_off = L.k_off;
  a.n_rows = L.n_rows;
  a.n_seq = L.n_seq;
  a.max_len = L.max_len;
  for (int i = 0; i < 32; ++i) a.inv_freq[i] = std::pow(L.theta, -2.0 * i / 64.0);
  a.q_out = L.q_out;
  a.w_out = L.w_out;
  a.k_cache = L.k_cache;
  a.err = L.err;
  e = launch_pdl(project_epilogue_kernel, dim3(L.n_rows), dim3(128), 0, st, a);
  count_launches(4);
  return e;
}

}  // namespace lsa
