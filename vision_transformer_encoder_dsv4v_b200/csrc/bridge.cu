// Image-token bridge into the language stream ([model-API, DeepseekV4Model]): the merge of
// aligner tokens and sentinel embeddings into the text embeddings (merge_image_embeddings) and
// the image-span visibility of the additive attention mask (apply_deepseek_v4_image_visibility).
//
// Pseudo-token types: -1 text, 0 image feature, 1 image_start, 2 image_end, 3 image_newline,
// 4 image_pad.  A span runs from an image_start to the next image_end of the same sequence and
// holds pseudo tokens only; every pseudo token lies inside one.
//
// Both calls start with the same two steps over chunks of kBridgeChunk positions: a count of
// features, starts and ends per chunk, then, per chunk, the exclusive prefix of those counts
// over the chunks before it plus a ballot scan inside the chunk.  That gives every position its
// feature index and its span index without any serial pass, and checks the span structure.
// The data movement that follows is bound by HBM:
//  * merge: each pseudo-token row is read once (aligner token or sentinel) and written once.
//    The pseudo rows of a batch gather in few chunks (images sit together in a sequence), so
//    every chunk is served by `slices` CTAs, each moving its own column slice of the rows from a
//    table of row addresses, eight 16-byte loads in flight per thread.  For a chunk of text
//    only, the CTA of slice 0 checks the layout and the others leave at once.  (Counting the
//    positions before each chunk inside the merge, by the CTAs of a cluster, saves the count
//    launch but measured slower on B200: 36.3 us against 32.2 us on the 16-image stream.)
//  * visibility: the scan records each span's first and last position; then one warp per mask
//    row writes the zeros of its span block with 16-byte stores.
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

constexpr int kTypeText = -1, kTypeImage = 0, kTypeStart = 1, kTypeEnd = 2, kTypePad = 4;
constexpr int kWarps = kBridgeChunk / 32;
constexpr int kBulkBufs = 4;                 // row buffers in flight per merge CTA (bulk mode)
constexpr size_t kBulkSmemMax = 160 * 1024;  // dynamic shared memory a bulk-mode merge CTA may take

__device__ __forceinline__ void record(uint32_t* err) { atomicCAS(err, 0u, static_cast<uint32_t>(kErrBridgeLayout)); }

// counts[c] = (features, image_starts, image_ends) among positions [c*kBridgeChunk, ...).  With
// span tables (visibility), also marks every span slot of this chunk's positions as unset.
__global__ void __launch_bounds__(kBridgeChunk) k_bridge_count(const int32_t* __restrict__ types, int64_t n,
                                                               int4* __restrict__ counts, int32_t* span_first,
                                                               int32_t* span_last, uint32_t* err) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t p = static_cast<int64_t>(blockIdx.x) * kBridgeChunk + threadIdx.x;
  const int t = p < n ? types[p] : kTypeText;
  if (t < kTypeText || t > kTypePad) record(err);
  if (span_first && p < n) {
    span_first[p] = -1;
    span_last[p] = -1;
  }
  const int c_img = __syncthreads_count(t == kTypeImage);
  const int c_start = __syncthreads_count(t == kTypeStart);
  const int c_end = __syncthreads_count(t == kTypeEnd);
  if (threadIdx.x == 0) counts[blockIdx.x] = make_int4(c_img, c_start, c_end, 0);
}

// What the scan tells one position of the chunk.
struct PosScan {
  int64_t p;            // position
  int t;                // its type (text past the end)
  int64_t k_img;        // features before p
  int64_t starts_incl;  // image_starts at or before p
  int64_t ends_excl;    // image_ends before p
  bool bad;             // violates the span structure
  int64_t total[3];     // features, starts, ends up to the end of this chunk
};

struct ScanSmem {
  int part[3][kWarps];
  int64_t base[3];  // features, starts, ends before the chunk
};

// sm.base from the per-chunk totals of the count launch.  All threads of the CTA must call it.
__device__ __forceinline__ void base_from_counts(const int4* __restrict__ counts, ScanSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    for (int k = 0; k < 3; ++k) sm.part[k][warp] = static_cast<int>(acc[k]);  // fewer than 2^31 positions
  __syncthreads();
  if (tid < 3) {
    int64_t s = 0;
    for (int w = 0; w < kWarps; ++w) s += sm.part[tid][w];
    sm.base[tid] = s;
  }
  __syncthreads();
}

// The ballot scan inside the chunk, from sm.base: checks that the type is known, that a
// sequence starts with every span closed, that text lies outside spans and that every other
// pseudo token lies inside exactly one.  Must be called by all threads of the CTA.
__device__ __forceinline__ PosScan chunk_scan(const int32_t* __restrict__ types, int64_t n, int64_t seq,
                                              ScanSmem& sm) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  PosScan r;
  r.p = static_cast<int64_t>(blockIdx.x) * kBridgeChunk + tid;
  r.t = r.p < n ? types[r.p] : kTypeText;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned b_img = __ballot_sync(0xffffffffu, r.t == kTypeImage);
  const unsigned b_st = __ballot_sync(0xffffffffu, r.t == kTypeStart);
  const unsigned b_en = __ballot_sync(0xffffffffu, r.t == kTypeEnd);
  if (lane == 0) {  // sm.part was last read before the base function's closing barrier
    sm.part[0][warp] = __popc(b_img);
    sm.part[1][warp] = __popc(b_st);
    sm.part[2][warp] = __popc(b_en);
  }
  __syncthreads();
  int64_t before[3] = {sm.base[0], sm.base[1], sm.base[2]};
  for (int k = 0; k < 3; ++k) r.total[k] = sm.base[k];
  for (int w = 0; w < kWarps; ++w)
    for (int k = 0; k < 3; ++k) {
      if (w < warp) before[k] += sm.part[k][w];
      r.total[k] += sm.part[k][w];
    }
  __syncthreads();  // sm.part is free again when this returns
  r.k_img = before[0] + __popc(b_img & lt);
  r.starts_incl = before[1] + __popc(b_st & (lt | (1u << lane)));
  r.ends_excl = before[2] + __popc(b_en & lt);
  const bool in_span = r.starts_incl - r.ends_excl == 1;
  r.bad = r.t < kTypeText || r.t > kTypePad;
  if (r.p < n) {
    if (r.p % seq == 0 && r.starts_incl - (r.t == kTypeStart) != r.ends_excl) r.bad = true;
    if (r.t == kTypeText ? in_span : !in_span) r.bad = true;
  }
  return r;
}

// grid (chunks, slices).  Every CTA of a chunk with pseudo tokens scans it; the one of slice 0
// reports layout errors (and is the only one to scan a chunk of text).  Each CTA then copies columns [s * vs,
// (s + 1) * vs) (16-byte vectors, vs = row_vec / slices) of the chunk's pseudo rows: aligner
// token rows for features, sentinel rows for the other pseudo types.
__global__ void __launch_bounds__(kBridgeChunk)
    k_bridge_merge(const int32_t* __restrict__ types, int64_t n, int64_t seq, const int4* __restrict__ counts,
                   const int32_t* __restrict__ grid, int n_images, int r, int64_t n_tokens,
                   const uint4* __restrict__ image_tokens, const uint4* __restrict__ sentinels,
                   uint4* __restrict__ embeds, int row_vec, int ring_off, uint32_t* err) {
  // Dynamic shared memory: [n_images + 1] aligner-token offsets of the images, then (bulk mode,
  // ring_off > 0) kBulkBufs row buffers at byte offset ring_off.
  extern __shared__ __align__(16) int32_t tok_cu[];
  __shared__ ScanSmem sm;
  __shared__ int warp_copies[kWarps];
  __shared__ int n_list;
  __shared__ __align__(8) uint64_t row_full[kBulkBufs];
  // The chunk's rows to copy, in position order: where this CTA's part of each row is read
  // (aligner token or sentinel) and written (a column slice, or the whole row in bulk mode).
  __shared__ const uint4* list_from[kBridgeChunk];
  __shared__ uint4* list_to[kBridgeChunk];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool bulk = ring_off > 0;
  grid_dependency_wait();
  launch_dependents();
  {
    // A chunk of text only copies nothing: slice 0 still scans it (the layout checks), the
    // other CTAs leave.
    const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kBridgeChunk + tid;
    const int t0 = p0 < n ? types[p0] : kTypeText;
    if (!__syncthreads_or(t0 != kTypeText) && blockIdx.y != 0) return;
  }

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
  base_from_counts(counts, sm);  // its barriers publish tok_cu
  const PosScan ps = chunk_scan(types, n, seq, sm);

  bool bad = ps.bad;
  int64_t s = -1;  // -1: keep the row
  if (!bad && ps.t != kTypeText && ps.p < n) {
    if (ps.t == kTypeImage) {
      const int64_t j = ps.starts_incl - 1;
      if (j >= n_images || ps.k_img < tok_cu[j] || ps.k_img >= tok_cu[j + 1]) bad = true;
      else s = ps.k_img;
    } else {
      s = -static_cast<int64_t>(ps.t) - 1;  // type 1..4 -> sentinel row 0..3
    }
  }
  if (blockIdx.y == 0) {
    if (bad) record(err);
    if (blockIdx.x == gridDim.x - 1 && tid == 0 &&
        (ps.total[0] != n_tokens || ps.total[1] != n_images || ps.total[1] != ps.total[2]))
      record(err);
  }
  // compact this chunk's rows to copy, in position order
  const bool copy = !bad && s != -1;
  const unsigned b_copy = __ballot_sync(0xffffffffu, copy);
  if (lane == 0) warp_copies[warp] = __popc(b_copy);
  __syncthreads();
  int slot = __popc(b_copy & ((1u << lane) - 1u));
  for (int w = 0; w < warp; ++w) slot += warp_copies[w];
  const int vs = bulk ? row_vec : row_vec / static_cast<int>(gridDim.y);
  const int col0 = bulk ? 0 : static_cast<int>(blockIdx.y) * vs;
  if (bulk && tid == 0) {
    for (int b = 0; b < kBulkBufs; ++b) mbar_init(&row_full[b], 1);
    fence_mbar_init();
  }
  if (copy) {
    list_from[slot] = (s >= 0 ? image_tokens + s * row_vec : sentinels + (-s - 2) * row_vec) + col0;
    list_to[slot] = embeds + ps.p * row_vec + col0;
  }
  if (tid == kBridgeChunk - 1) n_list = slot + (copy ? 1 : 0);
  __syncthreads();

  const int nl = n_list;
  if (bulk) {
    // Whole rows j = y, y + slices, ... of the chunk's list by bulk (TMA) copies through a ring of
    // kBulkBufs row buffers: one thread loads ahead, stores each row as it lands, and refills a
    // buffer once the store issued from it one row earlier has read it.
    if (tid != 0) return;
    const uint32_t rb = static_cast<uint32_t>(row_vec) * 16u;
    uint8_t* ring = reinterpret_cast<uint8_t*>(tok_cu) + ring_off;
    const int y = static_cast<int>(blockIdx.y), step = static_cast<int>(gridDim.y);
    const int mine = y < nl ? (nl - y + step - 1) / step : 0;
    for (int k = 0; k < mine && k < kBulkBufs; ++k) {
      mbar_arrive_expect_tx(&row_full[k], rb);
      bulk_load(ring + k * rb, list_from[y + k * step], rb, &row_full[k]);
    }
    volatile int never = 0;
    for (int k = 0; k < mine; ++k) {
      const int b = k % kBulkBufs;
      if (!mbar_wait(&row_full[b], static_cast<uint32_t>(k / kBulkBufs) & 1u, &never, err, kErrTimeoutProducer))
        break;
      bulk_store(list_to[y + k * step], ring + b * rb, rb);
      bulk_commit();
      const int kn = k - 1 + kBulkBufs;  // the next row of the previous row's buffer
      if (k >= 1 && kn < mine) {
        bulk_wait_read_1();  // every store but the one just issued has read its buffer
        const int bp = (k - 1) % kBulkBufs;
        mbar_arrive_expect_tx(&row_full[bp], rb);
        bulk_load(ring + bp * rb, list_from[y + kn * step], rb, &row_full[bp]);
      }
    }
    bulk_wait_all();
    return;
  }
  // Thread t copies vector column t % vs of rows t / vs, t / vs + rpp, ... (rpp rows per pass
  // of the CTA), eight independent 16-byte loads before their stores; no per-vector division.
  constexpr int kUnroll = 8;
  auto copy_rows = [&](int c, int r0, int step) {
    for (int j0 = r0; j0 < nl; j0 += step * kUnroll) {
      uint4 v[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = j0 + u * step;
        if (j < nl) v[u] = __ldg(list_from[j] + c);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int j = j0 + u * step;
        if (j < nl) list_to[j][c] = v[u];
      }
    }
  };
  if (vs <= kBridgeChunk) {
    const int rpp = kBridgeChunk / vs;
    const int r = tid / vs;
    if (r < rpp) copy_rows(tid - r * vs, r, rpp);
  } else {
    for (int c = tid; c < vs; c += kBridgeChunk) copy_rows(c, 0, 1);
  }
}

// Visibility, step 2: per chunk, the scan; each valid image_start / image_end stores its
// position in the span tables (index = span number), and every position its span number (-1
// for text or a bad position).
__global__ void __launch_bounds__(kBridgeChunk)
    k_span_scan(const int32_t* __restrict__ types, int64_t n, int64_t seq, const int4* __restrict__ counts,
                int32_t* __restrict__ span_first, int32_t* __restrict__ span_last, int32_t* __restrict__ span_of,
                uint32_t* err) {
  __shared__ ScanSmem sm;
  grid_dependency_wait();
  launch_dependents();
  base_from_counts(counts, sm);
  const PosScan ps = chunk_scan(types, n, seq, sm);
  if (ps.bad) record(err);
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0 && ps.total[1] != ps.total[2]) record(err);
  if (ps.p >= n) return;
  const bool pseudo = !ps.bad && ps.t != kTypeText;
  const int32_t j = static_cast<int32_t>(ps.starts_incl - 1);
  span_of[ps.p] = pseudo ? j : -1;
  if (pseudo && ps.t == kTypeStart) span_first[j] = static_cast<int32_t>(ps.p);
  if (pseudo && ps.t == kTypeEnd) span_last[j] = static_cast<int32_t>(ps.p);
}

// Visibility, step 3: one warp per mask row (b, i) of a pseudo token: zero the columns of its
// span, when both ends of the span were found inside the row's own sequence.
__global__ void __launch_bounds__(256)
    k_visibility_fill(const int32_t* __restrict__ span_of, const int32_t* __restrict__ span_first,
                      const int32_t* __restrict__ span_last, int64_t rows, int64_t seq, char* mask, int elem,
                      uint32_t* err) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int32_t j = span_of[row];
  if (j < 0) return;
  const int64_t a = span_first[j], e = span_last[j], lo = row - row % seq;
  if (a < lo || e >= lo + seq || a > row || e < row) {  // the span is not closed in this sequence
    if (lane == 0) record(err);
    return;
  }
  char* beg = mask + (row * seq + (a - lo)) * elem;
  char* end = mask + (row * seq + (e - lo) + 1) * elem;
  char* body = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(beg) + 15) & ~uintptr_t(15));
  if (body > end) body = end;
  char* tail = reinterpret_cast<char*>(reinterpret_cast<uintptr_t>(end) & ~uintptr_t(15));
  if (tail < body) tail = body;
  const int64_t head_n = (body - beg) / elem, tail_n = (end - tail) / elem;
  if (elem == 4) {
    for (int64_t k = lane; k < head_n; k += 32) reinterpret_cast<uint32_t*>(beg)[k] = 0u;
    for (int64_t k = lane; k < tail_n; k += 32) reinterpret_cast<uint32_t*>(tail)[k] = 0u;
  } else {
    for (int64_t k = lane; k < head_n; k += 32) reinterpret_cast<uint16_t*>(beg)[k] = 0;
    for (int64_t k = lane; k < tail_n; k += 32) reinterpret_cast<uint16_t*>(tail)[k] = 0;
  }
  const int64_t vecs = (tail - body) / 16;
  for (int64_t k = lane; k < vecs; k += 32) reinterpret_cast<uint4*>(body)[k] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

// CTAs per chunk of the merge: as many column slices of at least 32 vectors (one per lane) as
// divide the row, up to 16.
int bridge_slices(int row_vec) {
  int s = 1;
  while (s < 16 && row_vec % (2 * s) == 0 && row_vec / (2 * s) >= 32) s *= 2;
  return s;
}

cudaError_t launch_bridge_merge(const int32_t* types, int64_t n, int64_t seq, int4* counts, const int32_t* grid_dev,
                                int n_images, int r, int64_t n_tokens, const void* image_tokens, const void* sentinels,
                                void* embeds, int row_vec, uint32_t* err, cudaStream_t s) {
  const int64_t chunks = (n + kBridgeChunk - 1) / kBridgeChunk;
  if (chunks == 0) return cudaSuccess;
  cudaError_t e = launch_pdl(k_bridge_count, dim3(static_cast<unsigned>(chunks)), dim3(kBridgeChunk), 0, s, types, n,
                             counts, static_cast<int32_t*>(nullptr), static_cast<int32_t*>(nullptr), err);
  if (e != cudaSuccess) return e;
  // Rows of 2 KB or more move by bulk copies, whole rows per CTA (16 CTAs per chunk, each taking
  // every 16th row); narrower rows by 16-byte vectors, a column slice per CTA.
  const size_t row_bytes = static_cast<size_t>(row_vec) * 16;
  const size_t tok_bytes = (static_cast<size_t>(n_images) + 1) * sizeof(int32_t);
  const size_t ring_off = (tok_bytes + 127) / 128 * 128;
  const bool bulk = row_bytes >= 2048 && ring_off + kBulkBufs * row_bytes <= kBulkSmemMax;
  const size_t smem = bulk ? ring_off + kBulkBufs * row_bytes : tok_bytes;
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(k_bridge_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const int slices = bulk ? 16 : bridge_slices(row_vec);
  return launch_pdl(k_bridge_merge, dim3(static_cast<unsigned>(chunks), static_cast<unsigned>(slices)),
                    dim3(kBridgeChunk), smem, s, types, n, seq, static_cast<const int4*>(counts), grid_dev, n_images,
                    r, n_tokens, static_cast<const uint4*>(image_tokens), static_cast<const uint4*>(sentinels),
                    static_cast<uint4*>(embeds), row_vec, bulk ? static_cast<int>(ring_off) : 0, err);
}

cudaError_t launch_image_visibility(const int32_t* types, int64_t batch, int64_t seq, void* mask, int elem_bytes,
                                    int4* counts, int32_t* span_first, int32_t* span_last, int32_t* span_of,
                                    uint32_t* err, cudaStream_t s) {
  const int64_t n = batch * seq;
  const int64_t chunks = (n + kBridgeChunk - 1) / kBridgeChunk;
  if (chunks == 0) return cudaSuccess;
  cudaError_t e = launch_pdl(k_bridge_count, dim3(static_cast<unsigned>(chunks)), dim3(kBridgeChunk), 0, s, types, n,
                             counts, span_first, span_last, err);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_span_scan, dim3(static_cast<unsigned>(chunks)), dim3(kBridgeChunk), 0, s, types, n, seq,
                 static_cast<const int4*>(counts), span_first, span_last, span_of, err);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_visibility_fill, dim3(static_cast<unsigned>((n * 32 + 255) / 256)), dim3(256), 0, s,
                    static_cast<const int32_t*>(span_of), static_cast<const int32_t*>(span_first),
                    static_cast<const int32_t*>(span_last), n, seq, static_cast<char*>(mask), elem_bytes, err);
}

}  // namespace dsv4v
