// fp32 CUDA-core path of the block and aligner (tcgen05 has no exact-fp32 mode).  Used for
// DSV4V_F32 configs, which are small (vision_dim in the tens to hundreds).
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

constexpr int T = 32;  // output tile T x T, 256 threads, 4 outputs per thread

// out[M, n_out] = epi(A[M, K] . B[n, K]^T); SWIGLU uses B (gate) and B2 (up).
template <int EPI>
__global__ void __launch_bounds__(256) k_gemm_f32(const float* __restrict__ a, const float* __restrict__ b,
                                                  const float* __restrict__ b2, float* out,
                                                  const float* resid, int M, int n_out, int K,
                                                  const float* __restrict__ bias) {
  __shared__ float sa[T][T + 1];
  __shared__ float sb[T][T + 1];
  __shared__ float sb2[T][T + 1];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // ty in [0, 8)
  const int row0 = blockIdx.y * T, col0 = blockIdx.x * T;
  float acc[4] = {0, 0, 0, 0}, acc2[4] = {0, 0, 0, 0};
  for (int k0 = 0; k0 < K; k0 += T) {
    for (int i = ty; i < T; i += 8) {
      const int r = row0 + i, c = col0 + i, k = k0 + tx;
      sa[i][tx] = (r < M && k < K) ? a[static_cast<int64_t>(r) * K + k] : 0.0f;
      sb[i][tx] = (c < n_out && k < K) ? b[static_cast<int64_t>(c) * K + k] : 0.0f;
      if (EPI == EPI_SWIGLU) sb2[i][tx] = (c < n_out && k < K) ? b2[static_cast<int64_t>(c) * K + k] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < T; ++kk) {
      const float bv = sb[tx][kk];
      const float bv2 = EPI == EPI_SWIGLU ? sb2[tx][kk] : 0.0f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float av = sa[ty + 8 * q][kk];
        acc[q] = fmaf(av, bv, acc[q]);
        if (EPI == EPI_SWIGLU) acc2[q] = fmaf(av, bv2, acc2[q]);
      }
    }
    __syncthreads();
  }
  const int c = col0 + tx;
  if (c >= n_out) return;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int r = row0 + ty + 8 * q;
    if (r >= M) continue;
    const int64_t o = static_cast<int64_t>(r) * n_out + c;
    float v = acc[q];
    if (EPI == EPI_SWIGLU) v = acc[q] / (1.0f + expf(-acc[q])) * acc2[q];
    if (EPI == EPI_RESID) v += resid[o];
    if (EPI == EPI_STORE && bias) v += bias[c];
    if (EPI == EPI_GELU) {
      const float z = v + bias[c];
      v = 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
    }
    out[o] = v;
  }
}

// In-place half-split rotation of the q and k sections of qkv [P, 3D].
__global__ void k_rope_apply_f32(float* qkv, const float* __restrict__ cos, const float* __restrict__ sin, int64_t P,
                                 int d, int n_heads) {
  const int hd = d / n_heads, half = hd / 2;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_row = 2 * n_heads * half;  // q and k, every head, every pair
  if (idx >= P * per_row) return;
  const int64_t p = idx / per_row;
  int rem = static_cast<int>(idx - p * per_row);
  const int sec = rem / (n_heads * half);
  rem -= sec * n_heads * half;
  const int h = rem / half, j = rem - h * half;
  float* x = qkv + p * 3 * d + sec * d + h * hd;
  const float c = cos[p * half + j], s = sin[p * half + j];
  const float x1 = x[j], x2 = x[j + half];
  x[j] = x1 * c - x2 * s;
  x[j + half] = x2 * c + x1 * s;
}

// One thread per (packed query row, head): two passes over the keys of its image.
__global__ void k_attention_f32(const float* __restrict__ qkv, float* __restrict__ out,
                                const int32_t* __restrict__ cu, int n_images, int64_t P, int d, int n_heads) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= P * n_heads) return;
  const int64_t p = idx / n_heads;
  const int h = static_cast<int>(idx - p * n_heads);
  const int hd = d / n_heads;
  int lo = 0, hi = n_images - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= p) lo = mid;
    else hi = mid - 1;
  }
  const int64_t k0 = cu[lo], k1 = cu[lo + 1];
  const float* q = qkv + p * 3 * d + h * hd;
  const float scale = 1.0f / sqrtf(static_cast<float>(hd));
  float mx = -INFINITY;
  for (int64_t k = k0; k < k1; ++k) {
    const float* kr = qkv + k * 3 * d + d + h * hd;
    float s = 0.0f;
    for (int c = 0; c < hd; ++c) s = fmaf(q[c], kr[c], s);
    mx = fmaxf(mx, s * scale);
  }
  float acc[64];
  for (int c = 0; c < hd; ++c) acc[c] = 0.0f;
  float l = 0.0f;
  for (int64_t k = k0; k < k1; ++k) {
    const float* kr = qkv + k * 3 * d + d + h * hd;
    const float* vr = qkv + k * 3 * d + 2 * d + h * hd;
    float s = 0.0f;
    for (int c = 0; c < hd; ++c) s = fmaf(q[c], kr[c], s);
    const float e = expf(s * scale - mx);
    l += e;
    for (int c = 0; c < hd; ++c) acc[c] = fmaf(e, vr[c], acc[c]);
  }
  float* o = out + p * d + h * hd;
  for (int c = 0; c < hd; ++c) o[c] = acc[c] / l;
}

// merged[t, s * d + c] = x[src[t * r2 + s], c] (0 where src < 0).
__global__ void k_gather_f32(const float* __restrict__ x, const int32_t* __restrict__ src, float* __restrict__ merged,
                             int64_t n_tokens, int r2, int d) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= n_tokens * r2 * d) return;
  const int64_t t = idx / (static_cast<int64_t>(r2) * d);
  const int rem = static_cast<int>(idx - t * r2 * d);
  const int s = rem / d, c = rem - s * d;
  const int32_t row = src[t * r2 + s];
  merged[idx] = row >= 0 ? x[static_cast<int64_t>(row) * d + c] : 0.0f;
}

}  // namespace

cudaError_t launch_gemm_f32(int epi, const float* a, const float* b, const float* b2, float* out, const float* resid,
                            int M, int n_out, int K, cudaStream_t s, const float* bias) {
  if (M == 0) return cudaSuccess;
  dim3 grid((n_out + T - 1) / T, (M + T - 1) / T);
  switch (epi) {
    case EPI_STORE: k_gemm_f32<EPI_STORE><<<grid, 256, 0, s>>>(a, b, b2, out, resid, M, n_out, K, bias); break;
    case EPI_RESID: k_gemm_f32<EPI_RESID><<<grid, 256, 0, s>>>(a, b, b2, out, resid, M, n_out, K, nullptr); break;
    case EPI_SWIGLU: k_gemm_f32<EPI_SWIGLU><<<grid, 256, 0, s>>>(a, b, b2, out, resid, M, n_out, K, nullptr); break;
    case EPI_GELU: k_gemm_f32<EPI_GELU><<<grid, 256, 0, s>>>(a, b, b2, out, resid, M, n_out, K, bias); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_rope_apply_f32(float* qkv, const float* cos, const float* sin, int64_t P, int d, int n_heads,
                                  cudaStream_t s) {
  const int64_t n = P * d;  // 2 sections x n_heads x hd/2 pairs = d
  if (n == 0) return cudaSuccess;
  k_rope_apply_f32<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(qkv, cos, sin, P, d, n_heads);
  return cudaGetLastError();
}

cudaError_t launch_attention_f32(const float* qkv, float* out, const int32_t* cu_dev, int n_images, int64_t P,
                                 int d, int n_heads, cudaStream_t s) {
  const int64_t n = P * n_heads;
  if (n == 0) return cudaSuccess;
  k_attention_f32<<<static_cast<unsigned>((n + 127) / 128), 128, 0, s>>>(qkv, out, cu_dev, n_images, P, d, n_heads);
  return cudaGetLastError();
}

cudaError_t launch_gather_f32(const float* x, const int32_t* src, float* merged, int64_t n_tokens, int r2, int d,
                              cudaStream_t s) {
  const int64_t n = n_tokens * r2 * d;
  if (n == 0) return cudaSuccess;
  k_gather_f32<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(x, src, merged, n_tokens, r2, d);
  return cudaGetLastError();
}

}  // namespace dsv4v
