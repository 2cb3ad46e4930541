// Pieces shared by the tcgen05 GEMM kernels (the per-GEMM kernel and the persistent chain
// kernel): epilogue activations, the TMA-store staging of an epilogue warp, L2 loads and the
// bounded counter wait between CTAs.
#pragma once

#include "common.cuh"

namespace dsv4v {

// gelu(z) = z (1 + erf(z / sqrt 2)) / 2, the exact (erf) form.
__device__ __forceinline__ float gelu(float z) { return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f)); }

// silu(z) = z / (1 + e^-z) = (z / 2) (1 + tanh(z / 2)): one MUFU op per element, ample for a bf16
// result.
__device__ __forceinline__ float silu(float z) {
  const float h = 0.5f * z;
  return fmaf(h, tanh_approx(h), h);
}

// Output staging of one epilogue warp: two boxes of 32 rows x 128 bytes (64 bf16 columns) in
// the 128-byte-swizzled layout of the output tensor maps; lane i owns row i of a box.  Each box
// is written to global memory by one TMA store; a box is reused only after the store issued
// from it two stores ago has finished reading it.
struct Stager {
  uint8_t* base;
  int lane, n;
  __device__ __forceinline__ uint8_t* acquire() {
    if (lane == 0 && n >= 2) bulk_wait_read_1();
    __syncwarp();
    return base + (n & 1) * 4096;
  }
  // Both boxes, once no earlier store still reads either.
  __device__ __forceinline__ void acquire_both(uint8_t*& b0, uint8_t*& b1) {
    if (lane == 0 && n >= 1) bulk_wait_read_0();
    __syncwarp();
    b0 = base + (n & 1) * 4096;
    b1 = base + ((n + 1) & 1) * 4096;
  }
  // 16-byte chunk j (0..7) of this lane's row.
  __device__ __forceinline__ void put(uint8_t* box, int j, uint4 v) {
    *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
  }
  // Stores the box to rows [y, y + 32) and columns [x, x + 64) of `map` (TMA clips rows past
  // the end of the tensor; a box entirely past it is skipped).
  __device__ __forceinline__ void store(uint8_t* box, const CUtensorMap* map, int x, int y, int rows) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && y < rows) {
      tma_store_2d(map, box, x, y);
      bulk_commit();
    }
    ++n;
  }
  __device__ __forceinline__ void drain() {
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
};

__device__ __forceinline__ float4 ld_cg_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait until *ctr reaches `target` (the other contributors of a split tile, or the tiles
// an operand depends on); on timeout records `code`.
__device__ __forceinline__ bool wait_counter(const int* ctr, int target, volatile int* abort_flag, uint32_t* err,
                                             uint32_t code = kErrTimeoutEpilogue) {
  uint64_t t0 = 0;
  for (uint32_t i = 0;; ++i) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((i & 63u) == 63u) {
      if (*abort_flag) return false;
      const uint64_t now = global_timer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        atomicCAS(err, 0u, code);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Orders this thread's earlier generic-proxy accesses of global memory with its later
// async-proxy (TMA) accesses, and completed TMA stores with its later generic accesses.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

}  // namespace dsv4v
