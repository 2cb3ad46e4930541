// Image-token bridge into the language stream ([model-API, DeepseekV4Model]): the merge of
// aligner tokens and sentinel embeddings into the text embeddings (merge_image_embeddings) and
// the image-span visibility of the additive attention mask (apply_deepseek_v4_image_visibility).
//
// Pseudo-token types: -1 text, 0 image feature, 1 image_start, 2 image_end, 3 image_newline,
// 4 image_pad.  A span runs from an image_start to the next image_end of the same sequence;
// every other pseudo token lies inside one.  Both operations are copies, so they are bound by
// HBM: the merge moves each pseudo-token row once (read the source row, write the embedding
// row); the visibility call writes only the span blocks of the mask.
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

constexpr int kTypeText = -1, kTypeImage = 0, kTypeStart = 1, kTypeEnd = 2, kTypePad = 4;

__device__ __forceinline__ void record(uint32_t* err) { atomicCAS(err, 0u, static_cast<uint32_t>(kErrBridgeLayout)); }

// counts[c] = (features, image_starts, image_ends) among positions [c*kBridgeChunk, ...).
__global__ void __launch_bounds__(kBridgeChunk) k_bridge_count(const int32_t* __restrict__ types, int64_t n,
                                                               int4* __restrict__ counts, uint32_t* err) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t p = static_cast<int64_t>(blockIdx.x) * kBridgeChunk + threadIdx.x;
  const int t = p < n ? types[p] : kTypeText;
  if (t < kTypeText || t > kTypePad) record(err);
  const int c_img = __syncthreads_count(t == kTypeImage);
  const int c_start = __syncthreads_count(t == kTypeStart);
  const int c_end = __syncthreads_count(t == kTypeEnd);
  if (threadIdx.x == 0) counts[blockIdx.x] = make_int4(c_img, c_start, c_end, 0);
}

// One CTA per chunk of kBridgeChunk positions.  Each CTA rebuilds the exclusive prefix of the
// three counts over the chunks before it, scans its own chunk with warp ballots, checks the
// span structure and the per-image feature counts, then its warps copy the pseudo-token rows
// (row_vec 16-byte vectors each).
__global__ void __launch_bounds__(kBridgeChunk)
    k_bridge_merge(const int32_t* __restrict__ types, int64_t n, int64_t seq, const int4* __restrict__ counts,
                   const int32_t* __restrict__ grid, int n_images, int r, int64_t n_tokens,
                   const uint4* __restrict__ image_tokens, const uint4* __restrict__ sentinels, uint4* embeds,
                   int row_vec, uint32_t* err) {
  constexpr int kWarps = kBridgeChunk / 32;
  extern __shared__ int32_t tok_cu[];  // [n_images + 1] aligner-token offsets of the images
  __shared__ int part[3][kWarps];      // per-warp partial sums / counts
  __shared__ int64_t base[3];          // features, starts, ends before this chunk
  __shared__ int64_t src[kBridgeChunk];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dependency_wait();
  launch_dependents();

  if (warp == 0) {  // tok_cu by a warp-wide inclusive scan, 32 images at a time
    int carry = 0;
    if (lane == 0) tok_cu[0] = 0;
    for (int i0 = 0; i0 < n_images; i0 += 32) {
      const int i = i0 + lane;
      int v = 0;
      if (i < n_images) v = ((grid[2 * i] + r - 1) / r) * ((grid[2 * i + 1] + r - 1) / r);
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (i < n_images) tok_cu[i + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }

  // prefix over the previous chunks
  int64_t acc[3] = {0, 0, 0};
  for (int c = tid; c < static_cast<int>(blockIdx.x); c += kBridgeChunk) {
    const int4 v = counts[c];
    acc[0] += v.x;
    acc[1] += v.y;
    acc[2] += v.z;
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
  }
  if (lane == 0)
    for (int k = 0; k < 3; ++k) part[k][warp] = static_cast<int>(acc[k]);  // < 2^31 positions
  __syncthreads();
  if (tid < 3) {
    int64_t s = 0;
    for (int w = 0; w < kWarps; ++w) s += part[tid][w];
    base[tid] = s;
  }
  __syncthreads();

  // in-chunk scan
  const int64_t p = static_cast<int64_t>(blockIdx.x) * kBridgeChunk + tid;
  const int t = p < n ? types[p] : kTypeText;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned b_img = __ballot_sync(0xffffffffu, t == kTypeImage);
  const unsigned b_st = __ballot_sync(0xffffffffu, t == kTypeStart);
  const unsigned b_en = __ballot_sync(0xffffffffu, t == kTypeEnd);
  if (lane == 0) {
    part[0][warp] = __popc(b_img);
    part[1][warp] = __popc(b_st);
    part[2][warp] = __popc(b_en);
  }
  __syncthreads();
  int64_t before[3] = {base[0], base[1], base[2]};
  int64_t chunk_tot[3] = {0, 0, 0};
  for (int w = 0; w < kWarps; ++w)
    for (int k = 0; k < 3; ++k) {
      if (w < warp) before[k] += part[k][w];
      chunk_tot[k] += part[k][w];
    }
  const int64_t k_img = before[0] + __popc(b_img & lt);              // features before p
  const int64_t starts_incl = before[1] + __popc(b_st & (lt | (1u << lane)));  // starts at or before p
  const int64_t ends_excl = before[2] + __popc(b_en & lt);           // ends before p

  bool bad = t < kTypeText || t > kTypePad;
  // a sequence starts with every span closed
  if (p < n && p % seq == 0 && starts_incl - (t == kTypeStart) != ends_excl) bad = true;
  // a span holds pseudo tokens only
  if (p < n && t == kTypeText && starts_incl - ends_excl == 1) bad = true;
  int64_t s = -1;  // -1: keep the row; >= 0: aligner token; <= -2: sentinel row -s - 2
  if (!bad && t != kTypeText && p < n) {
    if (starts_incl - ends_excl != 1) {
      bad = true;  // outside a span, or a start inside an open one
    } else if (t == kTypeImage) {
      const int64_t j = starts_incl - 1;
      if (j >= n_images || k_img < tok_cu[j] || k_img >= tok_cu[j + 1]) bad = true;
      else s = k_img;
    } else {
      s = -static_cast<int64_t>(t) - 1;  // type 1..4 -> sentinel row 0..3
    }
  }
  if (bad) record(err);
  src[tid] = bad ? -1 : s;
  if (blockIdx.x == gridDim.x - 1 && tid == 0) {
    const int64_t f = base[0] + chunk_tot[0], st = base[1] + chunk_tot[1], en = base[2] + chunk_tot[2];
    if (f != n_tokens || st != n_images || st != en) record(err);
  }
  __syncthreads();

  for (int i = warp; i < kBridgeChunk; i += kWarps) {
    const int64_t si = src[i];
    if (si == -1) continue;
    const uint4* from = si >= 0 ? image_tokens + si * row_vec : sentinels + (-si - 2) * row_vec;
    uint4* to = embeds + (static_cast<int64_t>(blockIdx.x) * kBridgeChunk + i) * row_vec;
    int v = lane;
    for (; v + 96 < row_vec; v += 128) {
      const uint4 a0 = __ldg(from + v), a1 = __ldg(from + v + 32), a2 = __ldg(from + v + 64),
                  a3 = __ldg(from + v + 96);
      to[v] = a0;
      to[v + 32] = a1;
      to[v + 64] = a2;
      to[v + 96] = a3;
    }
    for (; v < row_vec; v += 32) to[v] = __ldg(from + v);
  }
}

// Nearest image_start / image_end at or before `from` (dir = -1) or at or after it (dir = +1)
// inside [lo, hi); returns its type, or kTypeText if there is none.  *text_between tells
// whether a text position lies between `from` and that marker (or the range's end).
__device__ __forceinline__ int nearest_marker(const int32_t* __restrict__ types, int64_t from, int dir, int64_t lo,
                                              int64_t hi, int64_t* at, bool* text_between) {
  const int lane = threadIdx.x & 31;
  bool text = false;
  for (int64_t q0 = from; q0 >= lo && q0 < hi; q0 += 32 * dir) {
    const int64_t q = q0 + dir * lane;
    const bool in = q >= lo && q < hi;
    const int t = in ? types[q] : kTypeText;
    const unsigned m = __ballot_sync(0xffffffffu, in && (t == kTypeStart || t == kTypeEnd));
    const unsigned tx = __ballot_sync(0xffffffffu, in && t == kTypeText);
    if (m) {
      const int first = __ffs(m) - 1;  // the lowest lane is the nearest position
      *at = q0 + dir * first;
      *text_between = text || (tx & ((1u << first) - 1u)) != 0;
      return __shfl_sync(0xffffffffu, t, first);
    }
    text = text || tx != 0;
  }
  *text_between = text;
  return kTypeText;
}

// One warp per mask row (b, i).  A pseudo token's span is bounded by the nearest image_start at
// or before it (strictly before an image_end) and the nearest image_end at or after it
// (strictly after an image_start); anything else is a layout error and the row is left as is.
// The image_start row also checks that no text lies inside its span.
template <typename E>
__global__ void __launch_bounds__(256) k_image_visibility(const int32_t* __restrict__ types, int64_t rows, int64_t seq,
                                                          E* mask, uint32_t* err) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int t = types[row];
  if (t == kTypeText) return;
  if (t < kTypeText || t > kTypePad) {
    if (lane == 0) record(err);
    return;
  }
  const int64_t lo = row - row % seq, hi = lo + seq;
  int64_t a = -1, e = -1;
  bool text_back, text_fwd;
  const int back = nearest_marker(types, t == kTypeEnd ? row - 1 : row, -1, lo, hi, &a, &text_back);
  const int fwd = nearest_marker(types, t == kTypeStart ? row + 1 : row, +1, lo, hi, &e, &text_fwd);
  if (back != kTypeStart || fwd != kTypeEnd || (t == kTypeStart && text_fwd)) {
    if (lane == 0) record(err);
    return;
  }
  E* out = mask + row * seq;  // columns are positions inside the sequence
  for (int64_t c = a - lo + lane; c <= e - lo; c += 32) out[c] = E(0);
}

}  // namespace

cudaError_t launch_bridge_merge(const int32_t* types, int64_t n, int64_t seq, int4* counts, const int32_t* grid_dev,
                                int n_images, int r, int64_t n_tokens, const void* image_tokens, const void* sentinels,
                                void* embeds, int row_vec, uint32_t* err, cudaStream_t s) {
  const int64_t chunks = (n + kBridgeChunk - 1) / kBridgeChunk;
  if (chunks == 0) return cudaSuccess;
  cudaError_t e = launch_pdl(k_bridge_count, dim3(static_cast<unsigned>(chunks)), dim3(kBridgeChunk), 0, s, types, n,
                             counts, err);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_bridge_merge, dim3(static_cast<unsigned>(chunks)), dim3(kBridgeChunk),
                    (n_images + 1) * sizeof(int32_t), s, types, n, seq, static_cast<const int4*>(counts), grid_dev,
                    n_images, r, n_tokens, static_cast<const uint4*>(image_tokens),
                    static_cast<const uint4*>(sentinels), static_cast<uint4*>(embeds), row_vec, err);
}

cudaError_t launch_image_visibility(const int32_t* types, int64_t batch, int64_t seq, void* mask, int elem_bytes,
                                    uint32_t* err, cudaStream_t s) {
  const int64_t rows = batch * seq;
  if (rows == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((rows * 32 + 255) / 256));
  if (elem_bytes == 4)
    return launch_pdl(k_image_visibility<uint32_t>, grid, dim3(256), 0, s, types, rows, seq,
                      static_cast<uint32_t*>(mask), err);
  return launch_pdl(k_image_visibility<uint16_t>, grid, dim3(256), 0, s, types, rows, seq,
                    static_cast<uint16_t*>(mask), err);
}

}  // namespace dsv4v
