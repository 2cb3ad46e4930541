// Memory-bound kernels of the path: the 2D rotary table, RMSNorm fused with the cast to the
// activation dtype, the aligner's window index table, and the bounded-wait self test.
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

// Block 0 clears n ints (the GEMM tile counters of the call).
__device__ __forceinline__ void zero_ints(int* ptr, int n) {
  if (ptr && blockIdx.x == 0)
    for (int i = threadIdx.x; i < n; i += blockDim.x) ptr[i] = 0;
}

// Index of the image that packed row p belongs to: largest i with cu[i] <= p.
__device__ __forceinline__ int image_of(const int32_t* cu, int n_images, int64_t p) {
  int lo = 0, hi = n_images - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= p) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// cos/sin [P, half]: column k < half/2 turns by the patch row h, column k >= half/2 by the
// patch column w, at inverse frequency theta^(-(k mod half/2) / (half/2)).
__global__ void k_rope_table(const int32_t* __restrict__ cu, const int32_t* __restrict__ grid, int n_images,
                             int64_t P, int half, float log2_theta, float* __restrict__ cos_out,
                             float* __restrict__ sin_out, int* zero_ptr, int zero_n) {
  grid_dependency_wait();
  launch_dependents();
  zero_ints(zero_ptr, zero_n);
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= P * half) return;
  const int64_t p = idx / half;
  const int k = static_cast<int>(idx - p * half);
  const int img = image_of(cu, n_images, p);
  const int local = static_cast<int>(p - cu[img]);
  const int n_w = grid[2 * img + 1];
  const int h = local / n_w, w = local - h * n_w;
  const int quarter = half >> 1;
  const int kk = k < quarter ? k : k - quarter;
  const float pos = static_cast<float>(k < quarter ? h : w);
  const float inv_freq = exp2f(-static_cast<float>(kk) / static_cast<float>(quarter) * log2_theta);
  float s, c;
  sincosf(pos * inv_freq, &s, &c);
  cos_out[idx] = c;
  sin_out[idx] = s;
}

// One warp per row (y may alias x).  Pass 1 accumulates the sum of squares in fp32; pass 2 re-reads the row
// (L1 hit), scales and casts.  bf16 rows are read and written 16 bytes per lane.
template <bool BF16>
__global__ void k_rmsnorm(const void* x, const float* __restrict__ w, void* y,
                          int64_t rows, int d, float eps, int* zero_ptr, int zero_n) {
  grid_dependency_wait();
  launch_dependents();
  zero_ints(zero_ptr, zero_n);
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float ss = 0.0f;
  if constexpr (BF16) {
    const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + row * d);
    for (int c = lane; c < d / 8; c += 32) {
      const uint4 v = xr[c];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = bf16_lo(u[e]), b = bf16_hi(u[e]);
        ss += a * a + b * b;
      }
    }
  } else {
    const float4* xr = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * d);
    for (int c = lane; c < d / 4; c += 32) {
      const float4 v = xr[c];
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
  if constexpr (BF16) {
    const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + row * d);
    uint4* yr = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) + row * d);
    const float4* w4 = reinterpret_cast<const float4*>(w);
    for (int c = lane; c < d / 8; c += 32) {
      const uint4 v = xr[c];
      const float4 wa = w4[2 * c], wb = w4[2 * c + 1];
      uint4 o;
      o.x = pack_bf16x2(bf16_lo(v.x) * inv * wa.x, bf16_hi(v.x) * inv * wa.y);
      o.y = pack_bf16x2(bf16_lo(v.y) * inv * wa.z, bf16_hi(v.y) * inv * wa.w);
      o.z = pack_bf16x2(bf16_lo(v.z) * inv * wb.x, bf16_hi(v.z) * inv * wb.y);
      o.w = pack_bf16x2(bf16_lo(v.w) * inv * wb.z, bf16_hi(v.w) * inv * wb.w);
      yr[c] = o;
    }
  } else {
    const float4* xr = reinterpret_cast<const float4*>(static_cast<const float*>(x) + row * d);
    float4* yr = reinterpret_cast<float4*>(static_cast<float*>(y) + row * d);
    const float4* w4 = reinterpret_cast<const float4*>(w);
    for (int c = lane; c < d / 4; c += 32) {
      const float4 v = xr[c], ww = w4[c];
      yr[c] = make_float4(v.x * inv * ww.x, v.y * inv * ww.y, v.z * inv * ww.z, v.w * inv * ww.w);
    }
  }
}

// First folded RMSNorm of a block (no residual GEMM precedes it): xw = bf16(x * w) and the row's
// sum of squares in ss[p * parts] (the remaining parts zero).  One warp per row, bf16 rows.
__global__ void k_norm_prep(const __nv_bfloat16* x, const float* __restrict__ w, __nv_bfloat16* xw, float* ss,
                            int parts, int64_t rows, int d, int* zero_ptr, int zero_n) {
  grid_dependency_wait();
  launch_dependents();
  zero_ints(zero_ptr, zero_n);
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * d);
  uint4* yr = reinterpret_cast<uint4*>(xw + row * d);
  const float4* w4 = reinterpret_cast<const float4*>(w);
  float acc = 0.0f;
  for (int c = lane; c < d / 8; c += 32) {
    const uint4 v = xr[c];
    const float4 wa = w4[2 * c], wb = w4[2 * c + 1];
    const float x0 = bf16_lo(v.x), x1 = bf16_hi(v.x), x2 = bf16_lo(v.y), x3 = bf16_hi(v.y);
    const float x4 = bf16_lo(v.z), x5 = bf16_hi(v.z), x6 = bf16_lo(v.w), x7 = bf16_hi(v.w);
    acc += ((x0 * x0 + x1 * x1) + (x2 * x2 + x3 * x3)) + ((x4 * x4 + x5 * x5) + (x6 * x6 + x7 * x7));
    uint4 o;
    o.x = pack_bf16x2(x0 * wa.x, x1 * wa.y);
    o.y = pack_bf16x2(x2 * wa.z, x3 * wa.w);
    o.z = pack_bf16x2(x4 * wb.x, x5 * wb.y);
    o.w = pack_bf16x2(x6 * wb.z, x7 * wb.w);
    yr[c] = o;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  for (int i = lane; i < parts; i += 32) ss[row * parts + i] = i == 0 ? acc : 0.0f;
}

// src[t * r^2 + a * r + b] = packed row of the patch at window position (a, b) of token t, or
// -1 where the window reaches into the zero padding.  Token offsets are rebuilt in shared
// memory from the grids (one prefix sum per block).
__global__ void k_aligner_index(const int32_t* __restrict__ cu, const int32_t* __restrict__ grid, int n_images,
                                int r, int64_t n_tokens, int32_t* __restrict__ src, int* zero_ptr, int zero_n) {
  extern __shared__ int32_t tok_cu[];  // [n_images + 1]
  grid_dependency_wait();
  launch_dependents();
  zero_ints(zero_ptr, zero_n);
  if (threadIdx.x == 0) {
    int32_t acc = 0;
    tok_cu[0] = 0;
    for (int i = 0; i < n_images; ++i) {
      const int g_h = (grid[2 * i] + r - 1) / r, g_w = (grid[2 * i + 1] + r - 1) / r;
      acc += g_h * g_w;
      tok_cu[i + 1] = acc;
    }
  }
  __syncthreads();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= n_tokens) return;
  const int img = image_of(tok_cu, n_images, t);
  const int n_h = grid[2 * img], n_w = grid[2 * img + 1];
  const int g_w = (n_w + r - 1) / r;
  const int local = static_cast<int>(t - tok_cu[img]);
  const int i = local / g_w, j = local - i * g_w;
  for (int a = 0; a < r; ++a)
    for (int b = 0; b < r; ++b) {
      const int h = r * i + a, w = r * j + b;
      src[t * r * r + a * r + b] = (h < n_h && w < n_w) ? cu[img] + h * n_w + w : -1;
    }
}

// One warp per (token, slot) row of the merged output: LayerNorm of the source patch row (mean
// and variance in fp32, two passes over the row), or zeros for a padding slot.
template <bool BF16>
__global__ void k_ln_merge(const void* __restrict__ x, const int32_t* __restrict__ src, const float* __restrict__ w,
                           const float* __restrict__ b, float eps, void* merged, int64_t n_rows, int d) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const int32_t s = src[row];
  auto in = [&](int c) -> float {
    if constexpr (BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(x)[static_cast<int64_t>(s) * d + c]);
    else return static_cast<const float*>(x)[static_cast<int64_t>(s) * d + c];
  };
  auto put = [&](int c, float v) {
    if constexpr (BF16) static_cast<__nv_bfloat16*>(merged)[row * d + c] = __float2bfloat16_rn(v);
    else static_cast<float*>(merged)[row * d + c] = v;
  };
  if (s < 0) {
    for (int c = lane; c < d; c += 32) put(c, 0.0f);
    return;
  }
  float sum = 0.0f;
  for (int c = lane; c < d; c += 32) sum += in(c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float mean = sum / static_cast<float>(d);
  float var = 0.0f;
  for (int c = lane; c < d; c += 32) {
    const float t = in(c) - mean;
    var += t * t;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) var += __shfl_xor_sync(0xffffffffu, var, o);
  const float inv = rsqrtf(var / static_cast<float>(d) + eps);
  for (int c = lane; c < d; c += 32) put(c, (in(c) - mean) * inv * w[c] + b[c]);
}

// One warp per (token, slot) row: a 16-byte-vector copy of the source patch row, or zeros.
__global__ void k_merge_rows_bf16(const uint4* __restrict__ x, const int32_t* __restrict__ src, uint4* merged,
                                  int64_t n_rows, int d8) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const int32_t s = src[row];
  uint4* dst = merged + row * d8;
  if (s < 0) {
    for (int c = lane; c < d8; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* in = x + static_cast<int64_t>(s) * d8;
  for (int c = lane; c < d8; c += 32) dst[c] = in[c];
}

// Clears the GEMM tile counters of a component call (one block; dependent launch, so that it
// costs no more than a kernel boundary inside a graph, unlike a memset node).
__global__ void k_zero_counters(int* ptr, int n) {
  grid_dependency_wait();
  launch_dependents();
  zero_ints(ptr, n);
}

// Waits on an mbarrier that nothing signals, with the production kernels' bounded wait.
__global__ void k_selftest_wait(uint64_t limit_ns, uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = global_timer_ns();
    bool done = false;
    while (!done) {
      if (mbar_try_wait(&bar, 0)) break;
      if (global_timer_ns() - t0 > limit_ns) {
        atomicCAS(err, 0u, static_cast<uint32_t>(kErrTimeoutSelftest));
        done = true;
      }
    }
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_rope_table(const int32_t* cu_dev, const int32_t* grid_dev, int n_images, int64_t P, int half,
                              float theta, float* cos_out, float* sin_out, cudaStream_t s, int* zero_ptr, int zero_n) {
  const int64_t n = P * half;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  return launch_pdl(k_rope_table, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, s, cu_dev, grid_dev,
                    n_images, P, half, log2f(theta), cos_out, sin_out, zero_ptr, zero_n);
}

cudaError_t launch_rmsnorm(bool bf16, const void* x, const float* w, void* y, int64_t rows, int d, float eps,
                           cudaStream_t s, int* zero_ptr, int zero_n) {
  if (rows == 0) return cudaSuccess;
  const int warps = 8;
  const unsigned blocks = static_cast<unsigned>((rows + warps - 1) / warps);
  if (bf16)
    return launch_pdl(k_rmsnorm<true>, dim3(blocks), dim3(warps * 32), 0, s, x, w, y, rows, d, eps, zero_ptr, zero_n);
  k_rmsnorm<false><<<blocks, warps * 32, 0, s>>>(x, w, y, rows, d, eps, zero_ptr, zero_n);
  return cudaGetLastError();
}

cudaError_t launch_norm_prep(const void* x, const float* w, void* xw, float* ss, int parts, int64_t rows, int d,
                             cudaStream_t s, int* zero_ptr, int zero_n) {
  if (rows == 0) return cudaSuccess;
  const int warps = 8;
  const unsigned blocks = static_cast<unsigned>((rows + warps - 1) / warps);
  return launch_pdl(k_norm_prep, dim3(blocks), dim3(warps * 32), 0, s, static_cast<const __nv_bfloat16*>(x), w,
                    static_cast<__nv_bfloat16*>(xw), ss, parts, rows, d, zero_ptr, zero_n);
}

cudaError_t launch_aligner_index(const int32_t* cu_dev, const int32_t* grid_dev, int n_images, int r,
                                 int64_t n_tokens, int32_t* src_out, cudaStream_t s, int* zero_ptr, int zero_n) {
  if (n_tokens == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n_tokens + threads - 1) / threads;
  return launch_pdl(k_aligner_index, dim3(static_cast<unsigned>(blocks)), dim3(threads),
                    (n_images + 1) * sizeof(int32_t), s, cu_dev, grid_dev, n_images, r, n_tokens, src_out, zero_ptr,
                    zero_n);
}

cudaError_t launch_ln_merge(bool bf16, const void* x, const int32_t* src, const float* w, const float* b, float eps,
                            void* merged, int64_t n_tokens, int r2, int d, cudaStream_t s) {
  const int64_t rows = n_tokens * r2;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows * 32 + 255) / 256;
  if (bf16) return launch_pdl(k_ln_merge<true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, x, src, w, b, eps,
                              merged, rows, d);
  return launch_pdl(k_ln_merge<false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, x, src, w, b, eps,
                    merged, rows, d);
}

cudaError_t launch_merge_rows_bf16(const void* x, const int32_t* src, void* merged, int64_t n_tokens, int r2, int d,
                                   cudaStream_t s) {
  const int64_t rows = n_tokens * r2;
  if (rows == 0) return cudaSuccess;
  const int64_t blocks = (rows * 32 + 255) / 256;
  return launch_pdl(k_merge_rows_bf16, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<const uint4*>(x), src, static_cast<uint4*>(merged), rows, d / 8);
}

cudaError_t launch_zero_counters(int* ptr, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  return launch_pdl(k_zero_counters, dim3(1), dim3(256), 0, s, ptr, n);
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, uint32_t* err, cudaStream_t s) {
  k_selftest_wait<<<1, 32, 0, s>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace dsv4v
