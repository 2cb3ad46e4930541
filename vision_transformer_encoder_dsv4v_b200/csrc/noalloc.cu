// dsv4v_linear_residual_noalloc: the residual GEMM (x <- x + a . w^T, bf16) for callers that
// cannot allocate device memory.  Every other entry point takes a caller-allocated workspace;
// this one keeps the split-tile scratch of the GEMM in a static device array of this library
// instead, so the caller passes only its inputs and outputs.
#include <mutex>

#include "dsv4v.h"
#include "internal.h"

namespace dsv4v {
dsv4v_status linear_residual_with_scratch(const dsv4v_config* cfg, int64_t rows, int k, const void* a,
                                          const void* w, void* x, float* partials, size_t partial_cap,
                                          int* counters, int counter_cap, void* stream);
}  // namespace dsv4v

namespace {

// Fixed scratch, allocated when the library is loaded and held by every GPU that loads it
// until the process exits: 10 MiB of fp32 split-tile partials (enough for 148 CTAs x a
// 128 x 128 tile) followed by 16384 tile counters.
constexpr size_t kPartialBytes = size_t(10) << 20;
constexpr int kCounters = 16384;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kPartialBytes + kCounters * sizeof(int)];

// Device address of g_noalloc_scratch, looked up once per device.  In host code the symbol
// itself is only a host-side handle, so the kernels get this address instead.
std::mutex g_mu;
void* g_addr[64] = {};

dsv4v_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSV4V_ERR_CUDA;
  if (dev < 0 || dev >= 64) return DSV4V_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSV4V_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return DSV4V_OK;
}

}  // namespace

extern "C" dsv4v_status dsv4v_linear_residual_noalloc(const dsv4v_config* cfg, int64_t rows, int k, const void* a,
                                                      const void* w, void* x, void* stream) {
  if (!cfg) return DSV4V_ERR_INVALID_ARG;
  if (rows > DSV4V_NOALLOC_MAX_ROWS) return DSV4V_ERR_UNSUPPORTED;
  void* base = nullptr;
  dsv4v_status st = scratch_address(&base);
  if (st != DSV4V_OK) return st;
  float* partials = static_cast<float*>(base);
  int* counters = reinterpret_cast<int*>(static_cast<unsigned char*>(base) + kPartialBytes);
  // The array keeps the previous call's contents; the tile counters the plan uses are cleared
  // on the stream after the call has been accepted, just before the GEMM.
  return dsv4v::linear_residual_with_scratch(cfg, rows, k, a, w, x, partials, kPartialBytes, counters, kCounters,
                                             stream);
}
