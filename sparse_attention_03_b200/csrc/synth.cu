// Synthetic inputs drawn on the device (tests and benchmarks only).
//
// Counter-based SplitMix64 (Steele, Lea and Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014): element i of the stream of
// tensor `tid` under `seed` is mix64(key + (i+1) * 0x9E3779B97F4A7C15) with
// key = mix64(seed ^ tid * 0xD1B54A32D192ED03). Normal element i sums the
// eight 16-bit fields of the stream's elements 2i and 2i+1 (Irwin-Hall, tails
// at about 4.9 sigma), centres the integer sum and multiplies it by one fp32
// constant; every step is exact or a single correctly rounded operation,
// so a host implementation of the same definition reproduces each value bit for
// bit.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace lsa {
namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kTidMul = 0xD1B54A32D192ED03ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ int fields16(uint64_t h) {
  return (int)(h & 0xFFFF) + (int)((h >> 16) & 0xFFFF) + (int)((h >> 32) & 0xFFFF) + (int)((h >> 48) & 0xFFFF);
}

__device__ __forceinline__ float normal_at(uint64_t key, int64_t i, float c) {
  const uint64_t h0 = mix64(key + (uint64_t)(2 * i + 1) * kGolden);
  const uint64_t h1 = mix64(key + (uint64_t)(2 * i + 2) * kGolden);
  const int s = fields16(h0) + fields16(h1) - 262140;  // |s| <= 262140: exact in fp32
  return __fmul_rn((float)s, c);
}

__global__ void synth_bf16_kernel(uint16_t* dst, int64_t n, uint64_t key, int64_t first, float c) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = f32_to_bf16_rne(normal_at(key, first + i, c));
}

__global__ void synth_f32_kernel(float* dst, int64_t n, uint64_t key, int64_t first, float c) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = normal_at(key, first + i, c);
}

// One warp per row of d values (d a multiple of 32, at most 1024).
__global__ void synth_rms_rows_kernel(uint16_t* dst, int64_t n_rows, int d, uint64_t key,
                                      int64_t first_row, float c) {
  const int lane = threadIdx.x & 31;
  const int per = d / 32;
  for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32; row < n_rows;
       row += ((int64_t)gridDim.x * blockDim.x) / 32) {
    float x[32];
    double ss = 0.0;
    for (int i = 0; i < per; ++i) {
      const int64_t e = (first_row + row) * d + lane + 32 * i;
      const uint16_t b = f32_to_bf16_rne(normal_at(key, e, c));
      x[i] = __uint_as_float((uint32_t)b << 16);
      ss += (double)x[i] * (double)x[i];  // exact: squares of bf16 values in fp64
    }
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const double rr = sqrt(ss / (double)d + 1e-6);
    for (int i = 0; i < per; ++i) {
      const float y = __double2float_rn((double)x[i] / rr);
      dst[row * d + lane + 32 * i] = f32_to_bf16_rne(y);
    }
  }
}

uint64_t stream_key(uint64_t seed, uint64_t tid) { return mix64(seed ^ (tid * kTidMul)); }

float normal_scale(double sigma) {
  return (float)(sigma / sqrt(2.0 * (65536.0 * 65536.0 - 1.0) / 3.0));
}

int grid_for(int64_t n, int threads) {
  const int64_t b = (n + threads - 1) / threads;
  return (int)(b < 148 * 16 ? (b < 1 ? 1 : b) : 148 * 16);
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" lsa_status lsa_synth_normal_bf16(lsa_bf16* dst, int64_t n, uint64_t seed, uint64_t tid,
                                            int64_t first, double sigma, void* stream) {
  if (!dst || n < 0 || first < 0) return set_error(LSA_ERR_INVALID, "lsa_synth_normal_bf16: bad arguments");
  if (n == 0) return LSA_OK;
  synth_bf16_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(
      dst, n, stream_key(seed, tid), first, normal_scale(sigma));
  count_launches(1);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LSA_OK : set_error(LSA_ERR_CUDA, "lsa_synth_normal_bf16: %s", cudaGetErrorString(e));
}

extern "C" lsa_status lsa_synth_normal_f32(float* dst, int64_t n, uint64_t seed, uint64_t tid,
                                           int64_t first, double sigma, void* stream) {
  if (!dst || n < 0 || first < 0) return set_error(LSA_ERR_INVALID, "lsa_synth_normal_f32: bad arguments");
  if (n == 0) return LSA_OK;
  synth_f32_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(
      dst, n, stream_key(seed, tid), first, normal_scale(sigma));
  count_launches(1);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LSA_OK : set_error(LSA_ERR_CUDA, "lsa_synth_normal_f32: %s", cudaGetErrorString(e));
}

extern "C" lsa_status lsa_synth_rms_rows_bf16(lsa_bf16* dst, int64_t n_rows, int32_t d, uint64_t seed,
                                              uint64_t tid, int64_t first_row, void* stream) {
  if (!dst || n_rows < 0 || first_row < 0 || d <= 0 || d % 32 != 0 || d > 1024)
    return set_error(LSA_ERR_INVALID, "lsa_synth_rms_rows_bf16: bad arguments");
  if (n_rows == 0) return LSA_OK;
  synth_rms_rows_kernel<<<grid_for(n_rows * 32, 256), 256, 0, (cudaStream_t)stream>>>(
      dst, n_rows, d, stream_key(seed, tid), first_row, normal_scale(1.0));
  count_launches(1);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LSA_OK : set_error(LSA_ERR_CUDA, "lsa_synth_rms_rows_bf16: %s", cudaGetErrorString(e));
}
