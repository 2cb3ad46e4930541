// Backward pass of the tower block ([PR], Validation: "ragged grids and backward"): the steps
// that are not GEMMs.  The weight and input gradients of the four projections run on the
// tcgen05 GEMM (api.cu), fed with transposed operands from k_transpose_bf16; this file holds the
// transposes, the RMSNorm and SwiGLU backward, the inverse rotation, and the attention backward.
//
// Attention backward, per image and head, with P = softmax(q k^T / sqrt(hd)) and o = P v:
//   dv = P^T do,  dS = P * (do v^T - rowsum(do * o)),  dq = dS k / sqrt(hd),  dk = dS^T q / sqrt(hd).
// Two kernels on 64 x 64 tiles in shared memory (fp32 math on bf16 inputs, CUDA cores):
//  * k_attn_bwd_dq: one CTA per (64-query block, head).  Pass 1 over the image's key blocks
//    finds each row's log-sum-exp; pass 2 rebuilds P, forms dS and accumulates dq.  It also
//    stores the log-sum-exp and rowsum(do * o) of its rows for the second kernel.
//  * k_attn_bwd_dkdv: one CTA per (64-key block, head): loops over the image's query blocks and
//    accumulates dk and dv.
// Neither kernel writes a location another CTA writes, so the result does not depend on the
// schedule.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

// ------------------------------------------------------------------------------ transpose
// out[c * ld_out + col0 + r] = in[r * ld_in + c] for r < rows, c < cols: a 32 x 32 tile per CTA
// through shared memory, so that both the reads and the writes run along rows.
__global__ void __launch_bounds__(256)
    k_transpose_bf16(const __nv_bfloat16* __restrict__ in, int64_t rows, int cols, int64_t ld_in,
                     __nv_bfloat16* __restrict__ out, int64_t ld_out, int64_t col0) {
  __shared__ __nv_bfloat16 tile[32][34];
  grid_dependency_wait();
  launch_dependents();
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * 32;
  const int c0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int64_t r = r0 + i;
    const int c = c0 + tx;
    if (r < rows && c < cols) tile[i][tx] = in[r * ld_in + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i;
    const int64_t r = r0 + tx;
    if (r < rows && c < cols) out[static_cast<int64_t>(c) * ld_out + col0 + r] = tile[tx][i];
  }
}

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
// g = dy * w, dx = r g - x r^3 (g . x) / d (+ d_in); the CTA's share of dw = sum dy * x * r is
// summed in shared memory and stored as partial[blockIdx.x][d].  d % 128 == 0.
__global__ void __launch_bounds__(256)
    k_rmsnorm_bwd(const __nv_bfloat16* __restrict__ x, const float* __restrict__ w, const __nv_bfloat16* dy,
                  const __nv_bfloat16* d_in, __nv_bfloat16* dx, float* __restrict__ partial, int64_t rows, int d,
                  float eps) {
  extern __shared__ float sdw[];  // [d]
  grid_dependency_wait();
  launch_dependents();
  for (int c = threadIdx.x; c < d; c += blockDim.x) sdw[c] = 0.0f;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
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
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        out[k] = r * dv[k] * wa[k] - xv[k] * coef + din[k];
        atomicAdd(&sdw[c + k], dv[k] * xv[k] * r);
      }
      store4(dx + row * d + c, out);
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x) partial[static_cast<int64_t>(blockIdx.x) * d + c] = sdw[c];
}

// out[c] = sum over p < parts of partial[p][c], in order.
__global__ void k_sum_parts(const float* __restrict__ partial, int parts, int d, float* __restrict__ out) {
  grid_dependency_wait();
  launch_dependents();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= d) return;
  float s = 0.0f;
  for (int p = 0; p < parts; ++p) s += partial[static_cast<int64_t>(p) * d + c];
  out[c] = s;
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
__global__ void __launch_bounds__(256)
    k_rotary_bwd(__nv_bfloat16* dqkv, const float* __restrict__ cos, const float* __restrict__ sin, int64_t P, int D,
                 int hd) {
  grid_dependency_wait();
  launch_dependents();
  const int half = hd / 2;
  const int64_t n = P * D;  // pairs: D per row (D / 2 in q, D / 2 in k)
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = i / D;
    const int j = static_cast<int>(i - p * D);
    const int part = j / (D / 2), jj = j - part * (D / 2);
    const int head = jj / half, e = jj - head * half;
    const int64_t col1 = p * 3 * D + part * D + head * hd + e;
    const float c = cos[p * half + e], s = sin[p * half + e];
    const float d1 = __bfloat162float(dqkv[col1]), d2 = __bfloat162float(dqkv[col1 + half]);
    dqkv[col1] = __float2bfloat16_rn(d1 * c + d2 * s);
    dqkv[col1 + half] = __float2bfloat16_rn(d2 * c - d1 * s);
  }
}

// ------------------------------------------------------------------------ attention backward
constexpr int kAB = 64;   // rows of a tile (queries or keys) and the head dim
constexpr int kLd = 68;   // shared-memory row stride in floats (16-byte rows for vector access)
constexpr int kTile = kAB * kLd;

// Block-count offsets of the images (ceil(N_i / 64) blocks each), by one warp; then the image
// of `item` and its block index inside the image.
__device__ __forceinline__ void image_blocks(const int32_t* __restrict__ cu, int n_images, int32_t* blk_cu) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    if (lane == 0) blk_cu[0] = 0;
    for (int i0 = 0; i0 < n_images; i0 += 32) {
      const int i = i0 + lane;
      int v = 0;
      if (i < n_images) v = (cu[i + 1] - cu[i] + kAB - 1) / kAB;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
      }
      if (i < n_images) blk_cu[i + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
}

__device__ __forceinline__ int image_of_block(const int32_t* blk_cu, int n_images, int item) {
  int lo = 0, hi = n_images - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (blk_cu[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Eight channels [col0 + 8v, col0 + 8v + 8) of row `row` (zeros past row_end), as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16* __restrict__ src, int64_t ld, int64_t row, int64_t row_end,
                                      int64_t col0, int v, float out[8]) {
  if (row < row_end) {
    const uint4 raw = *reinterpret_cast<const uint4*>(src + row * ld + col0 + v * 8);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      out[2 * k] = __low2float(h2[k]);
      out[2 * k + 1] = __high2float(h2[k]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) out[k] = 0.0f;
  }
}

// dst[r][c] = src[(row0 + r) * ld + col0 + c] for r < 64, c < 64, zero for rows >= row_end.
__device__ __forceinline__ void load_tile(float* dst, const __nv_bfloat16* __restrict__ src, int64_t ld, int64_t row0,
                                          int64_t row_end, int64_t col0) {
  for (int i = threadIdx.x; i < kAB * 8; i += blockDim.x) {
    const int r = i >> 3, v = i & 7;
    float f[8];
    load8(src, ld, row0 + r, row_end, col0, v, f);
    float4* d = reinterpret_cast<float4*>(dst + r * kLd + v * 8);
    d[0] = make_float4(f[0], f[1], f[2], f[3]);
    d[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}

// The transpose: dst[c][r] = src[(row0 + r) * ld + col0 + c].  Consecutive lanes take
// consecutive rows, so the shared-memory stores of a warp hit consecutive banks.
__device__ __forceinline__ void load_tile_t(float* dst, const __nv_bfloat16* __restrict__ src, int64_t ld,
                                            int64_t row0, int64_t row_end, int64_t col0) {
  for (int i = threadIdx.x; i < kAB * 8; i += blockDim.x) {
    const int r = i & (kAB - 1), v = i >> 6;
    float f[8];
    load8(src, ld, row0 + r, row_end, col0, v, f);
#pragma unroll
    for (int k = 0; k < 8; ++k) dst[(v * 8 + k) * kLd + r] = f[k];
  }
}

// acc[a][b] += sum over t < 64 of A(r0 + a, t) * B(t, s0 + b), with A(r, t) = A[r * ars + t * ats]
// and B(t, s) = B[t * bts + s] in shared memory.  B is read as one 16-byte vector per t (the 16
// column groups of a half-warp cover 256 contiguous bytes); A's four values are shared by the
// half-warp and broadcast.
__device__ __forceinline__ void mm64(const float* A, int ars, int ats, const float* B, int bts, int r0, int s0,
                                     float acc[4][4]) {
#pragma unroll 4
  for (int t = 0; t < kAB; ++t) {
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = A[(r0 + i) * ars + t * ats];
    const float4 bv = *reinterpret_cast<const float4*>(B + t * bts + s0);
    const float b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

__device__ __forceinline__ void zero44(float acc[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
}

struct AttnBwdArgs {
  const __nv_bfloat16* qkv;   // [P, 3D], q and k rotated (the attention's inputs)
  const __nv_bfloat16* out;   // [P, D], the attention's output
  const __nv_bfloat16* dout;  // [P, D]
  __nv_bfloat16* dqkv;        // [P, 3D], written
  float* lse;                 // [P, H]
  float* rowdot;              // [P, H], rowsum(do * o)
  const int32_t* cu;          // [n_images + 1]
  int n_images, D, H;
  float scale;                // 1 / sqrt(hd)
};

// Thread layout for 64 x 64 tiles: thread t owns rows r0..r0+3 (r0 = (t / 16) * 4) and columns
// s0..s0+3 (s0 = (t % 16) * 4); the 16 threads of a row group are 16 consecutive lanes.
__global__ void __launch_bounds__(256) k_attn_bwd_dq(AttnBwdArgs a) {
  extern __shared__ float sm[];
  float* sQ = sm;            // [query][channel]
  float* sDO = sQ + kTile;   // [query][channel]
  float* sKt = sDO + kTile;  // [channel][key]
  float* sVt = sKt + kTile;  // [channel][key]
  float* sK = sVt + kTile;   // [key][channel]
  float* sS = sK + kTile;    // [query][key]: dS
  float* sRowDot = sS + kTile;                              // [64]
  int32_t* blk_cu = reinterpret_cast<int32_t*>(sRowDot + kAB);  // [n_images + 1]
  grid_dependency_wait();
  launch_dependents();
  const int tid = threadIdx.x, r0 = (tid >> 4) * 4, s0 = (tid & 15) * 4;
  const int h = blockIdx.y, D = a.D, ld3 = 3 * a.D;
  image_blocks(a.cu, a.n_images, blk_cu);
  const int img = image_of_block(blk_cu, a.n_images, blockIdx.x);
  const int64_t beg = a.cu[img], end = a.cu[img + 1];
  const int64_t q0 = beg + static_cast<int64_t>(blockIdx.x - blk_cu[img]) * kAB;
  const int n_kb = static_cast<int>((end - beg + kAB - 1) / kAB);

  load_tile(sQ, a.qkv, ld3, q0, end, static_cast<int64_t>(h) * kAB);
  load_tile(sDO, a.dout, D, q0, end, static_cast<int64_t>(h) * kAB);
  load_tile(sS, a.out, D, q0, end, static_cast<int64_t>(h) * kAB);  // o, for rowsum(do * o)
  __syncthreads();
  if (tid < kAB) {
    float s = 0.0f;
    for (int c = 0; c < kAB; ++c) s += sDO[tid * kLd + c] * sS[tid * kLd + c];
    sRowDot[tid] = s;
  }
  __syncthreads();

  // pass 1: running max and sum of exp over the image's keys
  float m[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.0f;
  }
  for (int kb = 0; kb < n_kb; ++kb) {
    const int64_t k0 = beg + static_cast<int64_t>(kb) * kAB;
    load_tile_t(sKt, a.qkv, ld3, k0, end, D + static_cast<int64_t>(h) * kAB);
    __syncthreads();
    float acc[4][4];
    zero44(acc);
    mm64(sQ, kLd, 1, sKt, kLd, r0, s0, acc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (k0 + s0 + j < end) {
          const float s = acc[i][j] * a.scale;
          const float mn = fmaxf(m[i], s);
          l[i] = l[i] * expf(m[i] - mn) + expf(s - mn);
          m[i] = mn;
        }
    __syncthreads();
  }
  float lse[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m[i], o);
      const float l2 = __shfl_xor_sync(0xffffffffu, l[i], o);
      const float mn = fmaxf(m[i], m2);
      const float a1 = m[i] == -INFINITY ? 0.0f : l[i] * expf(m[i] - mn);
      const float a2 = m2 == -INFINITY ? 0.0f : l2 * expf(m2 - mn);
      m[i] = mn;
      l[i] = a1 + a2;
    }
    lse[i] = m[i] + logf(l[i]);
  }

  // pass 2: P, dS and dq
  float dq[4][4];
  zero44(dq);
  for (int kb = 0; kb < n_kb; ++kb) {
    const int64_t k0 = beg + static_cast<int64_t>(kb) * kAB;
    load_tile_t(sKt, a.qkv, ld3, k0, end, D + static_cast<int64_t>(h) * kAB);
    load_tile_t(sVt, a.qkv, ld3, k0, end, 2 * D + static_cast<int64_t>(h) * kAB);
    load_tile(sK, a.qkv, ld3, k0, end, D + static_cast<int64_t>(h) * kAB);
    __syncthreads();
    float s[4][4], dp[4][4];
    zero44(s);
    zero44(dp);
    mm64(sQ, kLd, 1, sKt, kLd, r0, s0, s);
    mm64(sDO, kLd, 1, sVt, kLd, r0, s0, dp);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float ds[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float p = k0 + s0 + j < end ? expf(s[i][j] * a.scale - lse[i]) : 0.0f;
        ds[j] = p * (dp[i][j] - sRowDot[r0 + i]);
      }
      *reinterpret_cast<float4*>(sS + (r0 + i) * kLd + s0) = make_float4(ds[0], ds[1], ds[2], ds[3]);
    }
    __syncthreads();
    mm64(sS, kLd, 1, sK, kLd, r0, s0, dq);
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = q0 + r0 + i;
    if (row >= end) continue;
    float v[4] = {dq[i][0] * a.scale, dq[i][1] * a.scale, dq[i][2] * a.scale, dq[i][3] * a.scale};
    store4(a.dqkv + row * ld3 + static_cast<int64_t>(h) * kAB + s0, v);
    if (s0 == 0) {
      a.lse[row * a.H + h] = lse[i];
      a.rowdot[row * a.H + h] = sRowDot[r0 + i];
    }
  }
}

__global__ void __launch_bounds__(256) k_attn_bwd_dkdv(AttnBwdArgs a) {
  extern __shared__ float sm[];
  float* sKt = sm;            // [channel][key]
  float* sVt = sKt + kTile;   // [channel][key]
  float* sQ = sVt + kTile;    // [query][channel]
  float* sDO = sQ + kTile;    // [query][channel]
  float* sP = sDO + kTile;    // [query][key]
  float* sDS = sP + kTile;    // [query][key]
  float* sLse = sDS + kTile;                                // [64]
  float* sRowDot = sLse + kAB;                              // [64]
  int32_t* blk_cu = reinterpret_cast<int32_t*>(sRowDot + kAB);  // [n_images + 1]
  grid_dependency_wait();
  launch_dependents();
  const int tid = threadIdx.x, r0 = (tid >> 4) * 4, s0 = (tid & 15) * 4;
  const int h = blockIdx.y, D = a.D, ld3 = 3 * a.D;
  image_blocks(a.cu, a.n_images, blk_cu);
  const int img = image_of_block(blk_cu, a.n_images, blockIdx.x);
  const int64_t beg = a.cu[img], end = a.cu[img + 1];
  const int64_t k0 = beg + static_cast<int64_t>(blockIdx.x - blk_cu[img]) * kAB;
  const int n_qb = static_cast<int>((end - beg + kAB - 1) / kAB);

  load_tile_t(sKt, a.qkv, ld3, k0, end, D + static_cast<int64_t>(h) * kAB);
  load_tile_t(sVt, a.qkv, ld3, k0, end, 2 * D + static_cast<int64_t>(h) * kAB);
  float dk[4][4], dv[4][4];
  zero44(dk);
  zero44(dv);
  for (int qb = 0; qb < n_qb; ++qb) {
    const int64_t q0 = beg + static_cast<int64_t>(qb) * kAB;
    load_tile(sQ, a.qkv, ld3, q0, end, static_cast<int64_t>(h) * kAB);
    load_tile(sDO, a.dout, D, q0, end, static_cast<int64_t>(h) * kAB);
    if (tid < kAB) {
      const int64_t row = q0 + tid;
      sLse[tid] = row < end ? a.lse[row * a.H + h] : 0.0f;
      sRowDot[tid] = row < end ? a.rowdot[row * a.H + h] : 0.0f;
    }
    __syncthreads();
    float s[4][4], dp[4][4];
    zero44(s);
    zero44(dp);
    mm64(sQ, kLd, 1, sKt, kLd, r0, s0, s);    // rows: queries, columns: keys
    mm64(sDO, kLd, 1, sVt, kLd, r0, s0, dp);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float pv[4], ds[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool ok = q0 + r0 + i < end && k0 + s0 + j < end;
        pv[j] = ok ? expf(s[i][j] * a.scale - sLse[r0 + i]) : 0.0f;
        ds[j] = pv[j] * (dp[i][j] - sRowDot[r0 + i]);
      }
      *reinterpret_cast<float4*>(sP + (r0 + i) * kLd + s0) = make_float4(pv[0], pv[1], pv[2], pv[3]);
      *reinterpret_cast<float4*>(sDS + (r0 + i) * kLd + s0) = make_float4(ds[0], ds[1], ds[2], ds[3]);
    }
    __syncthreads();
    mm64(sP, 1, kLd, sDO, kLd, r0, s0, dv);   // rows: keys, columns: channels
    mm64(sDS, 1, kLd, sQ, kLd, r0, s0, dk);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = k0 + r0 + i;
    if (row >= end) continue;
    float vk[4] = {dk[i][0] * a.scale, dk[i][1] * a.scale, dk[i][2] * a.scale, dk[i][3] * a.scale};
    float vv[4] = {dv[i][0], dv[i][1], dv[i][2], dv[i][3]};
    store4(a.dqkv + row * ld3 + D + static_cast<int64_t>(h) * kAB + s0, vk);
    store4(a.dqkv + row * ld3 + 2 * D + static_cast<int64_t>(h) * kAB + s0, vv);
  }
}

}  // namespace

cudaError_t launch_transpose_bf16(const void* in, int64_t rows, int cols, int64_t ld_in, void* out, int64_t ld_out,
                                  int64_t col0, cudaStream_t s) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((cols + 31) / 32), static_cast<unsigned>((rows + 31) / 32));
  return launch_pdl(k_transpose_bf16, grid, dim3(256), 0, s, static_cast<const __nv_bfloat16*>(in), rows, cols, ld_in,
                    static_cast<__nv_bfloat16*>(out), ld_out, col0);
}

cudaError_t launch_rmsnorm_bwd(const void* x, const float* w, const void* dy, const void* d_in, void* dx,
                               float* partial, int parts, float* dw, int64_t rows, int d, float eps, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(d) * sizeof(float);
  cudaError_t e = launch_pdl(k_rmsnorm_bwd, dim3(static_cast<unsigned>(parts)), dim3(256), smem, s,
                             static_cast<const __nv_bfloat16*>(x), w, static_cast<const __nv_bfloat16*>(dy),
                             static_cast<const __nv_bfloat16*>(d_in), static_cast<__nv_bfloat16*>(dx), partial, rows, d,
                             eps);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_sum_parts, dim3(static_cast<unsigned>((d + 255) / 256)), dim3(256), 0, s,
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
  const int64_t n = P * D;
  if (n == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n + 255) / 256, static_cast<int64_t>(sms) * 8);
  return launch_pdl(k_rotary_bwd, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                    static_cast<__nv_bfloat16*>(dqkv), cos, sin, P, D, hd);
}

size_t attn_bwd_smem(int kernel, int n_images) {
  const size_t tiles = 6;
  const size_t vecs = kernel == 0 ? 1 : 2;
  return tiles * kTile * sizeof(float) + vecs * kAB * sizeof(float) + (n_images + 1) * sizeof(int32_t);
}

cudaError_t launch_attention_bwd(const void* qkv, const void* out, const void* dout, void* dqkv, float* lse,
                                 float* rowdot, const int32_t* cu_dev, int n_images, int total_blocks, int D, int H,
                                 cudaStream_t s) {
  if (total_blocks == 0) return cudaSuccess;
  AttnBwdArgs a;
  a.qkv = static_cast<const __nv_bfloat16*>(qkv);
  a.out = static_cast<const __nv_bfloat16*>(out);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.dqkv = static_cast<__nv_bfloat16*>(dqkv);
  a.lse = lse;
  a.rowdot = rowdot;
  a.cu = cu_dev;
  a.n_images = n_images;
  a.D = D;
  a.H = H;
  a.scale = 1.0f / sqrtf(static_cast<float>(D / H));
  const size_t smem0 = attn_bwd_smem(0, n_images), smem1 = attn_bwd_smem(1, n_images);
  cudaError_t e = cudaFuncSetAttribute(k_attn_bwd_dq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem0));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(k_attn_bwd_dkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem1));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(total_blocks), static_cast<unsigned>(H));
  e = launch_pdl(k_attn_bwd_dq, grid, dim3(256), smem0, s, a);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_attn_bwd_dkdv, grid, dim3(256), smem1, s, a);
}

}  // namespace dsv4v
