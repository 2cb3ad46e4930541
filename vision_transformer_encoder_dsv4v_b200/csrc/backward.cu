// Backward pass of the tower block ([PR], Validation: "ragged grids and backward"): the steps
// that are neither GEMMs nor attention.  The weight and input gradients of the four projections
// run on the tcgen05 GEMM (api.cu), which reads the activations, gradients and weights where
// they lie (MN-major operands where needed); the attention backward is attn_bwd_tc.cu; this
// file holds the RMSNorm and SwiGLU backward and the inverse rotation.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

// ------------------------------------------------------------------------- RMSNorm backward
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float v[4]) {
  const uint2 raw = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  v[0] = __low2float(a);
  v[1] = __high2float(a);
  v[2] = __low2float(b);
  v[3] = __high2float(b);
}

__device__ __forceinline__ void store4(__nv_bfloat16* p, const float v[4]) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
  uint2 raw;
  raw.x = *reinterpret_cast<const uint32_t*>(&a);
  raw.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = raw;
}

// y = w * x * r, r = 1 / sqrt(mean(x^2) + eps).  One warp per row (grid-stride): with
// g = dy * w, dx = r g - x r^3 (g . x) / d (+ d_in).  dw = sum dy * x * r: each warp adds its
// rows' terms into its own row of shared memory (no atomics, no contention), then the CTA sums
// the warps' rows in warp order into partial[blockIdx.x][d].  d % 128 == 0.
__global__ void __launch_bounds__(256)
    k_rmsnorm_bwd(const __nv_bfloat16* __restrict__ x, const float* __restrict__ w, const __nv_bfloat16* dy,
                  const __nv_bfloat16* d_in, __nv_bfloat16* dx, float* __restrict__ partial, int64_t rows, int d,
                  float eps) {
  extern __shared__ float sdw[];  // [warps][d]
  grid_dependency_wait();
  launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
  float* my = sdw + static_cast<size_t>(warp) * d;
  for (int c = lane * 4; c < d; c += 128) *reinterpret_cast<float4*>(my + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * n_warps + warp; row < rows;
       row += static_cast<int64_t>(gridDim.x) * n_warps) {
    const __nv_bfloat16* xr = x + row * d;
    const __nv_bfloat16* dyr = dy + row * d;
    float ss = 0.0f, dot = 0.0f;
    for (int c = lane * 4; c < d; c += 128) {
      float xv[4], gv[4];
      load4(xr + c, xv);
      load4(dyr + c, gv);
      const float4 wv = *reinterpret_cast<const float4*>(w + c);
      ss += xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
      dot += gv[0] * wv.x * xv[0] + gv[1] * wv.y * xv[1] + gv[2] * wv.z * xv[2] + gv[3] * wv.w * xv[3];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      dot += __shfl_xor_sync(0xffffffffu, dot, o);
    }
    const float r = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
    const float coef = r * r * r * dot / static_cast<float>(d);
    for (int c = lane * 4; c < d; c += 128) {
      float xv[4], dv[4], out[4];
      load4(xr + c, xv);
      load4(dyr + c, dv);
      const float4 wv = *reinterpret_cast<const float4*>(w + c);
      const float wa[4] = {wv.x, wv.y, wv.z, wv.w};
      float din[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      if (d_in) load4(d_in + row * d + c, din);
      float4 acc = *reinterpret_cast<const float4*>(my + c);
      acc.x += dv[0] * xv[0] * r;
      acc.y += dv[1] * xv[1] * r;
      acc.z += dv[2] * xv[2] * r;
      acc.w += dv[3] * xv[3] * r;
      *reinterpret_cast<float4*>(my + c) = acc;
#pragma unroll
      for (int k = 0; k < 4; ++k) out[k] = r * dv[k] * wa[k] - xv[k] * coef + din[k];
      store4(dx + row * d + c, out);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float t = 0.0f;
    for (int wi = 0; wi < n_warps; ++wi) t += sdw[static_cast<size_t>(wi) * d + c];
    partial[static_cast<int64_t>(blockIdx.x) * d + c] = t;
  }
}

// out[c] = sum over p < parts of partial[p][c] in a fixed order: warp y of a CTA of 8 warps
// sums parts y, y + 8, y + 16, ... of 32 consecutive columns (coalesced), then the 8 warp sums
// are added in warp order.  Deterministic.
__global__ void __launch_bounds__(256) k_sum_parts(const float* __restrict__ partial, int parts, int d,
                                                   float* __restrict__ out) {
  __shared__ float part_sum[8][32];
  grid_dependency_wait();
  launch_dependents();
  const int lane = threadIdx.x & 31, wy = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  float t = 0.0f;
  if (c < d)
    for (int p = wy; p < parts; p += 8) t += partial[static_cast<int64_t>(p) * d + c];
  part_sum[wy][lane] = t;
  __syncthreads();
  if (wy == 0 && c < d) {
    float v = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) v += part_sum[k][lane];
    out[c] = v;
  }
}

// -------------------------------------------------------------------------- SwiGLU backward
// h = silu(g) * u.  dg = dh * u * silu'(g), du = dh * silu(g) into dgu = [dg | du] (row width
// 2f); also h itself (the input of the down projection).  f % 4 == 0.
__global__ void __launch_bounds__(256)
    k_swiglu_bwd(const __nv_bfloat16* __restrict__ g, const __nv_bfloat16* __restrict__ u,
                 const __nv_bfloat16* __restrict__ dh, __nv_bfloat16* __restrict__ dgu, __nv_bfloat16* __restrict__ h,
                 int64_t rows, int f) {
  grid_dependency_wait();
  launch_dependents();
  const int per_row = f / 4;
  const int64_t n = rows * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / per_row;
    const int c = static_cast<int>(i - row * per_row) * 4;
    float gv[4], uv[4], dv[4], dg[4], du[4], hv[4];
    load4(g + row * f + c, gv);
    load4(u + row * f + c, uv);
    load4(dh + row * f + c, dv);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float sg = 1.0f / (1.0f + expf(-gv[k]));
      const float silu = gv[k] * sg;
      dg[k] = dv[k] * uv[k] * sg * (1.0f + gv[k] * (1.0f - sg));
      du[k] = dv[k] * silu;
      hv[k] = silu * uv[k];
    }
    store4(dgu + row * 2 * f + c, dg);
    store4(dgu + row * 2 * f + f + c, du);
    store4(h + row * f + c, hv);
  }
}

// ------------------------------------------------------------------------ inverse rotation
// In place on the q and k columns of dqkv [P, 3D]: each half-split pair (j, j + hd/2) of a head
// is turned back by its angle: (d1, d2) <- (d1 c + d2 s, d2 c - d1 s).  cos/sin: [P, hd/2].
// One thread per row and 8 consecutive pairs of one head (16-byte loads of each half; hd/2 is
// a multiple of 8), CTAs striding over the rows.
__global__ void __launch_bounds__(256)
    k_rotary_bwd(__nv_bfloat16* dqkv, const float* __restrict__ cos, const float* __restrict__ sin, int64_t P, int D,
                 int hd) {
  grid_dependency_wait();
  launch_dependents();
  const int half = hd / 2;
  const int groups = D / 8;  // per row: D / 2 pairs in q and D / 2 in k, 8 per group
  const int per_part = groups / 2;
  for (int64_t p = blockIdx.x; p < P; p += gridDim.x) {
    for (int gi = threadIdx.x; gi < groups; gi += blockDim.x) {
      const int part = gi >= per_part ? 1 : 0;
      const int jj0 = (gi - part * per_part) * 8;
      const int head = jj0 / half, e0 = jj0 - head * half;
      __nv_bfloat16* a = dqkv + p * 3 * D + part * D + head * hd + e0;
      const uint4 ra = *reinterpret_cast<const uint4*>(a);
      const uint4 rb = *reinterpret_cast<const uint4*>(a + half);
      const float4 c0 = *reinterpret_cast<const float4*>(cos + p * half + e0);
      const float4 c1 = *reinterpret_cast<const float4*>(cos + p * half + e0 + 4);
      const float4 s0 = *reinterpret_cast<const float4*>(sin + p * half + e0);
      const float4 s1 = *reinterpret_cast<const float4*>(sin + p * half + e0 + 4);
      const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const __nv_bfloat16* va = reinterpret_cast<const __nv_bfloat16*>(&ra);
      const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(&rb);
      uint4 oa, ob;
      __nv_bfloat16* wa = reinterpret_cast<__nv_bfloat16*>(&oa);
      __nv_bfloat16* wb = reinterpret_cast<__nv_bfloat16*>(&ob);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float d1 = __bfloat162float(va[k]), d2 = __bfloat162float(vb[k]);
        wa[k] = __float2bfloat16_rn(d1 * cs[k] + d2 * sn[k]);
        wb[k] = __float2bfloat16_rn(d2 * cs[k] - d1 * sn[k]);
      }
      *reinterpret_cast<uint4*>(a) = oa;
      *reinterpret_cast<uint4*>(a + half) = ob;
    }
  }
}

}  // namespace

cudaError_t launch_rmsnorm_bwd(const void* x, const float* w, const void* dy, const void* d_in, void* dx,
                               float* partial, int parts, float* dw, int64_t rows, int d, float eps, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(d) * sizeof(float) * 8;  // one row of dw per warp
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  static int attr_dev = -1;
  if (smem > 48 * 1024) {
    int dev = 0;
    cudaError_t ea = cudaGetDevice(&dev);
    if (ea != cudaSuccess) return ea;
    if (attr_dev != dev) {
      ea = cudaFuncSetAttribute(k_rmsnorm_bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
      if (ea != cudaSuccess) return ea;
      attr_dev = dev;
    }
  }
  cudaError_t e = launch_pdl(k_rmsnorm_bwd, dim3(static_cast<unsigned>(parts)), dim3(256), smem, s,
                             static_cast<const __nv_bfloat16*>(x), w, static_cast<const __nv_bfloat16*>(dy),
                             static_cast<const __nv_bfloat16*>(d_in), static_cast<__nv_bfloat16*>(dx), partial, rows, d,
                             eps);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_sum_parts, dim3(static_cast<unsigned>((d + 31) / 32)), dim3(256), 0, s,
                    static_cast<const float*>(partial), parts, d, dw);
}

cudaError_t launch_swiglu_bwd(const void* g, const void* u, const void* dh, void* dgu, void* h, int64_t rows, int f,
                              int sms, cudaStream_t s) {
  const int64_t n = rows * (f / 4);
  if (n == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(sms) * 8);
  return launch_pdl(k_swiglu_bwd, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<const __nv_bfloat16*>(g), static_cast<const __nv_bfloat16*>(u),
                    static_cast<const __nv_bfloat16*>(dh), static_cast<__nv_bfloat16*>(dgu),
                    static_cast<__nv_bfloat16*>(h), rows, f);
}

cudaError_t launch_rotary_bwd(void* dqkv, const float* cos, const float* sin, int64_t P, int D, int hd, int sms,
                              cudaStream_t s) {
  if (P == 0) return cudaSuccess;
  if (D % 16 || (hd / 2) % 8) return cudaErrorInvalidValue;
  const int threads = std::min(256, (D / 8 + 31) / 32 * 32);
  const int64_t blocks = std::min<int64_t>(P, static_cast<int64_t>(sms) * 8);
  return launch_pdl(k_rotary_bwd, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, s,
                    static_cast<__nv_bfloat16*>(dqkv), cos, sin, P, D, hd);
}

}  // namespace dsv4v
