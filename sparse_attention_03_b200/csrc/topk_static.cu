// lsa_topk_static: the top-k of lsa_topk, with its scratch memory in a
// fixed-size array that lives in the library instead of a caller workspace.
//
// Some callers cannot allocate device memory at the point where they select:
// code being recorded into a CUDA graph (an allocation is not a stream
// operation and breaks or is refused by the capture), serving loops that must
// never pay the implicit device synchronisation that cudaMalloc/cudaFree can
// cause, and plugins that a host framework hands only their input and output
// buffers. This entry point needs nothing but those buffers.
//
// The scratch is a file-scope __device__ array sized for
// LSA_TOPK_STATIC_MAX_ROWS rows. Every GPU that loads the library holds it
// until the process exits. Host code cannot use the array's name as a device
// address, so the device address is looked up once per device with
// cudaGetSymbolAddress on the first call made while that device is current.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace lsa {
namespace {

constexpr int kStaticRows = LSA_TOPK_STATIC_MAX_ROWS;

static __device__ __align__(256) unsigned char g_topk_scratch[(size_t)kStaticRows * kTopkRowBytes];

// Device address of g_topk_scratch on the current device (null on failure).
// Host threads may make their first calls on a device at the same time: each
// then looks the address up and stores the same value, through atomics.
void* static_scratch() {
  static std::atomic<void*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* p = addr[dev].load(std::memory_order_relaxed);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess) return nullptr;
    addr[dev].store(p, std::memory_order_relaxed);
  }
  return p;
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" lsa_status lsa_topk_static(const lsa_config* c, int32_t n_rows, const int32_t* pos,
                                      int64_t max_len, const float* scores, int64_t ld, int32_t* idx,
                                      int32_t* count, void* stream) {
  const char* fn = "lsa_topk_static";
  const lsa_status cs = check_cfg(c, fn);  // the same configurations as lsa_topk
  if (cs != LSA_OK) return cs;
  if (n_rows < 0 || max_len < 1 || ld < max_len)
    return set_error(LSA_ERR_INVALID, "%s: need n_rows >= 0 and 1 <= max_len <= ld", fn);
  if (n_rows > kStaticRows)
    return set_error(LSA_ERR_INVALID,
                     "%s: %d rows exceed the built-in scratch of %d rows; split the call or use lsa_topk", fn,
                     n_rows, kStaticRows);
  if (n_rows == 0) return max_len <= c->index_topk ? LSA_DENSE : LSA_OK;
  if (!pos || !scores || !idx || !count) return set_error(LSA_ERR_INVALID, "%s: NULL array argument", fn);
  void* ws = static_scratch();
  if (!ws) return set_error(LSA_ERR_CUDA, "%s: cannot resolve the scratch array's device address", fn);
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.pos = pos;
  a.n_rows = n_rows;
  a.max_len = max_len;
  a.topk = c->index_topk;
  a.n_init = c->index_init_tokens;
  a.n_loc = c->index_local_tokens;
  a.idx = idx;
  a.count = count;
  a.ws = ws;
  a.ws_bytes = (size_t)kStaticRows * kTopkRowBytes;
  // launch_topk clears the histogram/control block of every row before use, so
  // what a previous call left in the array does not matter.
  const cudaError_t e = launch_topk(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return set_error(LSA_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
  return max_len <= c->index_topk ? LSA_DENSE : LSA_OK;
}
