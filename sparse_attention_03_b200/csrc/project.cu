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
// (angles in fp64: positions reach ~10^6), writes the bf16 query, the fp32 head
// weights and the bf16 key row into the cache at the row's position.
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
__global__ void __launch_bounds__(kGemmThreads) gemm_tn_kernel(const uint16_t* __restrict__ x,
                                                               const uint16_t* __restrict__ w, float* __restrict__ out,
                                                               int M, int N, int K) {
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
  const int n_kt = K / kBK;
  load(0, 0);
  cp_async_commit();
  for (int kt = 0; kt < n_kt; ++kt) {
    const int st = kt & 1;
    if (kt + 1 < n_kt) load(kt + 1, st ^ 1);
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
        if (col < N) out[(int64_t)row * N + col] = acc[nt][2 * hf];
        if (col + 1 < N) out[(int64_t)row * N + col + 1] = acc[nt][2 * hf + 1];
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
  double theta;
  uint16_t* q_out;       // [rows, 32, 128] bf16
  float* w_out;          // [rows, 32]
  uint16_t* k_cache;     // packed [sum L, 128] bf16
  int* err;
};

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

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
    const int i = (d - (kDi - 64)) & 31;
    const double ang = (double)p * pow(a.theta, -2.0 * i / 64.0);
    c = (float)cos(ang);
    s = (float)sin(ang);
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

}  // namespace

size_t project_ws_bytes(int n_rows) { return (size_t)n_rows * (kHi * kDi + kDi + kHi) * sizeof(float) + 256; }

cudaError_t launch_index_project(const ProjectLaunch& L, cudaStream_t st) {
  if (L.n_rows <= 0) return cudaSuccess;
  float* q = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(L.ws) + 255) & ~uintptr_t(255));
  float* k = q + (size_t)L.n_rows * kHi * kDi;
  float* wh = k + (size_t)L.n_rows * kDi;
  const int my = (L.n_rows + kBM - 1) / kBM;
  if (my > 65535) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(gemm_tn_kernel, dim3(kHi * kDi / kBN, my), dim3(kGemmThreads), 0, st, L.c_q, L.wq_b, q,
                             L.n_rows, kHi * kDi, L.q_lora);
  if (e != cudaSuccess) return e;
  e = launch_pdl(gemm_tn_kernel, dim3(kDi / kBN, my), dim3(kGemmThreads), 0, st, L.hidden, L.wk, k, L.n_rows, kDi,
                 L.hidden_dim);
  if (e != cudaSuccess) return e;
  e = launch_pdl(gemm_tn_kernel, dim3(1, my), dim3(kGemmThreads), 0, st, L.hidden, L.wproj, wh, L.n_rows, kHi,
                 L.hidden_dim);
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
  a.theta = L.theta;
  a.q_out = L.q_out;
  a.w_out = L.w_out;
  a.k_cache = L.k_cache;
  a.err = L.err;
  e = launch_pdl(project_epilogue_kernel, dim3(L.n_rows), dim3(128), 0, st, a);
  count_launches(4);
  return e;
}

}  // namespace lsa
