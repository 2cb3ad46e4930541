// Persistent multi-stage tcgen05 GEMM ("chain kernel") for batches of a few thousand patches or
// fewer, where every GEMM of the block is only one wave of output tiles and per-launch ramps and
// tails, not the tensor pipe, set the time.
//
// One launch runs several dependent GEMM stages of the block back to back, e.g. the output
// projection (+ residual, prepares norm2), the SwiGLU gate/up GEMM (norm2 folded in), the down
// projection (+ residual, prepares the next norm1) and the next block's fused q|k|v projection
// (+ 2D rotary).  The stages' tiles form one ticket sequence: stage by stage, row tile by row
// tile, column tile, K split.  Each CTA (one per SM, persistent) repeatedly takes the next ticket
// from a global counter, so CTAs take work in ticket order and the split-K contributors of a
// tile hold consecutive tickets.
//
// Dependencies are per 128-row tile: a stage that reads the output of an earlier stage of the
// same launch waits until that stage has finished every column tile of the row tile (a counter
// per row tile, released by the tile's finisher after its stores are complete).  A split tile
// is finished by its last split, which waits for the earlier splits' fp32 partials and adds
// them in split order (deterministic).  Every wait is on a smaller ticket, and a CTA handles its
// tickets in increasing order, so the waits cannot form a cycle; CTAs that are not yet resident
// hold no tickets, so nothing waits on them.
//
// Warp roles (192 threads, as the per-GEMM kernel):
//   warp 0     ticket taker + TMA producer: the weight tiles of a task's first stages are
//              requested before its dependency wait, the activation tiles after it
//   warp 1     TMEM owner + single-thread tcgen05.mma issuer (M = 128, N = task's BN)
//   warps 2-5  epilogue: split-K partials, fused epilogue math, TMA stores, completion release
// Tasks pass from the producer to the other roles through a small ring of descriptors in shared
// memory.  The fp32 accumulator is double-buffered in TMEM (2 x 256 columns).
#include "common.cuh"
#include "internal.h"
#include "tile_util.cuh"

namespace dsv4v {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
// Operand ring: kRingBytes split into ChainParams::ring_slots slots of slot_bytes (the launch's
// largest stage, A + B of one K block), at most kRingMax of them.
constexpr int kRingBytes = 208 * 1024;
constexpr int kRingMax = 8;
constexpr int kABytes = BM * BK * 2;
constexpr int kStagingBytes = 4 * 4096;       // per epilogue warp: one 32-row x 64-column bf16 box
constexpr int kTaskSlots = 4;
constexpr int kThreads = 192;
constexpr int OFF_STAGING = kRingBytes;
constexpr int OFF_BAR = OFF_STAGING + kStagingBytes;
constexpr int kBarBytes = 1024;
constexpr int SMEM = 1024 + OFF_BAR + kBarBytes;
constexpr int kAccCols = 256;                 // TMEM columns per accumulator buffer
static_assert(SMEM <= 232448, "shared memory budget");

struct Task {
  int stage, m, n, split, kb0, kb1, done, pad;
};

__device__ __forceinline__ void decode(const ChainParams& p, int t, Task& k) {
  int s = 0;
  while (s + 1 < p.n_stages && t >= p.st[s + 1].task_base) ++s;
  const ChainStage& d = p.st[s];
  const int local = t - d.task_base;
  const int per_m = d.tiles_n * d.splits;
  k.stage = s;
  k.m = local / per_m;
  const int r = local - k.m * per_m;
  k.n = r / d.splits;
  k.split = r - k.n * d.splits;
  k.kb0 = k.split * d.kb_total / d.splits;
  k.kb1 = (k.split + 1) * d.kb_total / d.splits;
  k.done = 0;
  k.pad = 0;
}

// 1 / sqrt(mean x^2 + eps) of output row `row` from the partial sums of squares that the stage
// producing the norm's operand wrote (1 when the stage has no norm folded in).
__device__ __forceinline__ float chain_row_scale(const ChainParams& p, const ChainStage& d, int row) {
  if (!d.norm_ss) return 1.0f;
  const float* s = d.norm_ss + static_cast<size_t>(min(row, d.M - 1)) * d.norm_stride;
  float acc = 0.0f;
  for (int i = 0; i < d.norm_parts; ++i) acc += s[i];
  return 1.0f / sqrtf(acc * p.norm_inv_d + p.norm_eps);
}

// Adds the fp32 partials of the earlier splits of this tile (split order) to accumulator chunks
// c0 and c1 (32 columns each) of this thread's row.
__device__ __forceinline__ void add_partials(const ChainStage& d, int tile, int row_in_tile, int c0, int c1,
                                             float (&v)[64]) {
  for (int s = 0; s + 1 < d.splits; ++s) {
    const float* src = d.partials + (static_cast<size_t>(tile) * (d.splits - 1) + s) * BM * d.bn;
    float4 a[8], b[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      a[q] = ld_cg_f4(src + ((c0 * 8 + q) * BM + row_in_tile) * 4);
      b[q] = ld_cg_f4(src + ((c1 * 8 + q) * BM + row_in_tile) * 4);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      v[4 * q + 0] += a[q].x;
      v[4 * q + 1] += a[q].y;
      v[4 * q + 2] += a[q].z;
      v[4 * q + 3] += a[q].w;
      v[32 + 4 * q + 0] += b[q].x;
      v[32 + 4 * q + 1] += b[q].y;
      v[32 + 4 * q + 2] += b[q].z;
      v[32 + 4 * q + 3] += b[q].w;
    }
  }
}

// wait_counter with a short pause between polls: many CTAs poll the same counters, and each
// poll is an L2 round trip.
__device__ __forceinline__ bool wait_counter_backoff(const int* ctr, int target, volatile int* abort_flag,
                                                     uint32_t* err, uint32_t code) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    __nanosleep(64);
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((i & 15u) == 0) {
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

__device__ __forceinline__ void load_acc(uint32_t t_row, int c0, int c1, float (&v)[64]) {
  uint32_t r0[32], r1[32];
  tmem_ld32(t_row + c0 * 32, r0);
  tmem_ld32(t_row + c1 * 32, r1);
  tmem_ld_wait(r0);
  tmem_ld_wait(r1);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    v[j] = __uint_as_float(r0[j]);
    v[32 + j] = __uint_as_float(r1[j]);
  }
}

// Output staging of one epilogue warp: one box of 32 rows x 64 bf16 columns in the 128-byte
// swizzled layout of the output tensor maps (lane i owns row i); each box goes out by one TMA
// store and is reused once that store has read it.
struct Stager1 {
  uint8_t* box;
  int lane, n;
  __device__ __forceinline__ uint8_t* acquire() {
    if (lane == 0 && n >= 1) bulk_wait_read_0();
    __syncwarp();
    return box;
  }
  __device__ __forceinline__ void put(int j, uint4 v) {
    *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
  }
  __device__ __forceinline__ void store(const CUtensorMap* map, int x, int y, int rows) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && y < rows) {
      tma_store_2d(map, box, x, y);
      bulk_commit();
    }
    ++n;
  }
};

__device__ __forceinline__ void pack8(const float* v, uint4 (&o)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    o[q].x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    o[q].y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    o[q].z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    o[q].w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
  }
}

// One task of the epilogue warps.  The inputs of the epilogue math (folded-norm row scale,
// rotation tables, residual row) are fetched before the accumulator is waited for, so that their
// L2 round trips overlap the MMAs.  An earlier split parks its fp32 partial; the finisher adds
// the partials (split order), runs the epilogue math, stores, and releases the row tile's counter
// once its stores are complete.
//   CHAIN_RESID: x <- x + acc on columns [n BN, (n + 1) BN), optionally also bf16(x * w) and the
//     row's partial sum of x^2 over these columns.
//   CHAIN_SWIGLU: accumulator = gate columns then up columns of output columns
//     [n BN/2, (n + 1) BN/2); h = silu(r gate) * (r up), r the folded norm's row scale.
//   CHAIN_QKV_HEADS: accumulator = the q, k and v columns of head n (64 each); rows scaled by r,
//     q and k rotated, each 64-column group stored at column g D + 64 n.
// Returns false when a bounded wait gave up.
template <int EPI>
__device__ __forceinline__ bool epilogue_task(const ChainParams& p, const ChainStage& d, const Task& k,
                                              uint32_t t_row, uint64_t* tfull_acc, uint64_t* tempty_acc,
                                              uint32_t acc_phase, int quad, int lane, int et, Stager1& st,
                                              volatile int* abort_flag, volatile int* ticket_ok) {
  const int row_in_tile = quad * 32 + lane;
  const int row = k.m * BM + row_in_tile;
  const int prow = min(row, d.M - 1);
  const int box_y = k.m * BM + quad * 32;
  const int tile = k.m * d.tiles_n + k.n;
  const bool finisher = k.split + 1 == d.splits;
  const int ngroups = d.bn / 64;
  // ---- inputs fetched while the MMAs run
  float scale = 1.0f;
  float rc[EPI == CHAIN_QKV_HEADS ? 32 : 1], rs[EPI == CHAIN_QKV_HEADS ? 32 : 1];
  uint4 res[EPI == CHAIN_RESID ? 16 : 1];  // residual: the first two 64-column groups
  const uint4* rrow = nullptr;
  if (finisher) {
    if constexpr (EPI != CHAIN_RESID) {
      scale = chain_row_scale(p, d, row);
      pin(scale);
    }
    if constexpr (EPI == CHAIN_QKV_HEADS) {
      const float4* c4 = reinterpret_cast<const float4*>(d.cos + static_cast<size_t>(prow) * 32);
      const float4* s4 = reinterpret_cast<const float4*>(d.sin + static_cast<size_t>(prow) * 32);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 c = c4[q], sv = s4[q];
        rc[4 * q] = c.x; rc[4 * q + 1] = c.y; rc[4 * q + 2] = c.z; rc[4 * q + 3] = c.w;
        rs[4 * q] = sv.x; rs[4 * q + 1] = sv.y; rs[4 * q + 2] = sv.z; rs[4 * q + 3] = sv.w;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        pin(rc[j]);
        pin(rs[j]);
      }
    }
    if constexpr (EPI == CHAIN_RESID) {
      rrow = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(d.resid) +
                                            static_cast<size_t>(prow) * d.ldr + k.n * d.bn);
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (q < 8 * ngroups) res[q] = rrow[q];
#pragma unroll
      for (int q = 0; q < 16; ++q) pin(res[q]);
    }
  }
  const bool got = mbar_wait(tfull_acc, acc_phase, abort_flag, p.err, kErrTimeoutEpilogue);
  if (!named_barrier_and(2, 128, got)) return false;
  tc_fence_after_sync();
  if (!finisher) {
    // An earlier split of the tile: park the fp32 partial, release it, move on.
    float* part = d.partials + (static_cast<size_t>(tile) * (d.splits - 1) + k.split) * BM * d.bn;
    for (int c = 0; c < d.bn / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(t_row + c * 32, r);
      tmem_ld_wait(r);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        *reinterpret_cast<float4*>(part + ((c * 8 + q) * BM + row_in_tile) * 4) =
            make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                        __uint_as_float(r[4 * q + 3]));
    }
    tc_fence_before_sync();
    mbar_arrive(tempty_acc);
    __threadfence();
    named_barrier_sync(1, 128);
    if (et == 0) atomicAdd(d.arrivals + tile, 1);
    return true;
  }
  if (d.splits > 1) {
    if (et == 0)
      *ticket_ok = wait_counter_backoff(d.arrivals + tile, d.splits - 1, abort_flag, p.err, kErrTimeoutEpilogue) ? 1
                                                                                                                 : 0;
    named_barrier_sync(1, 128);
    if (!*ticket_ok) {
      tc_fence_before_sync();
      mbar_arrive(tempty_acc);
      return false;
    }
    __threadfence();
  }
  const CUtensorMap* m_out = &p.maps[d.map_out];
  if constexpr (EPI == CHAIN_RESID) {
    const CUtensorMap* m_xw = d.map_xw >= 0 ? &p.maps[d.map_xw] : nullptr;
    float ss_acc = 0.0f;
    // Group g uses the residual slot r (8 x 16 bytes: 64 columns), refilled two groups ahead.
    auto group = [&](int g, uint4* r) {
      float v[64];
      load_acc(t_row, 2 * g, 2 * g + 1, v);
      add_partials(d, tile, row_in_tile, 2 * g, 2 * g + 1, v);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 x = r[q];
        v[8 * q + 0] += bf16_lo(x.x);
        v[8 * q + 1] += bf16_hi(x.x);
        v[8 * q + 2] += bf16_lo(x.y);
        v[8 * q + 3] += bf16_hi(x.y);
        v[8 * q + 4] += bf16_lo(x.z);
        v[8 * q + 5] += bf16_hi(x.z);
        v[8 * q + 6] += bf16_lo(x.w);
        v[8 * q + 7] += bf16_hi(x.w);
      }
      if (g + 2 < ngroups) {
#pragma unroll
        for (int q = 0; q < 8; ++q) r[q] = rrow[8 * (g + 2) + q];
      }
      uint4 o[8];
      pack8(v, o);
      st.acquire();
#pragma unroll
      for (int q = 0; q < 8; ++q) st.put(q, o[q]);
      st.store(m_out, k.n * d.bn + g * 64, box_y, d.M);
      if (m_xw) {
        // The next norm's operand from the stored (bf16) x: bf16(x * w) and the sum of x^2.
        const float4* w4 = reinterpret_cast<const float4*>(d.xw_w + k.n * d.bn + g * 64);
        st.acquire();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 wa = w4[2 * q], wb = w4[2 * q + 1];
          const float x0 = bf16_lo(o[q].x), x1 = bf16_hi(o[q].x), x2 = bf16_lo(o[q].y), x3 = bf16_hi(o[q].y);
          const float x4 = bf16_lo(o[q].z), x5 = bf16_hi(o[q].z), x6 = bf16_lo(o[q].w), x7 = bf16_hi(o[q].w);
          ss_acc += ((x0 * x0 + x1 * x1) + (x2 * x2 + x3 * x3)) + ((x4 * x4 + x5 * x5) + (x6 * x6 + x7 * x7));
          uint4 t;
          t.x = pack_bf16x2(x0 * wa.x, x1 * wa.y);
          t.y = pack_bf16x2(x2 * wa.z, x3 * wa.w);
          t.z = pack_bf16x2(x4 * wb.x, x5 * wb.y);
          t.w = pack_bf16x2(x6 * wb.z, x7 * wb.w);
          st.put(q, t);
        }
        st.store(m_xw, k.n * d.bn + g * 64, box_y, d.M);
      }
    };
    for (int g = 0; g < ngroups; g += 2) {
      group(g, res);
      if (g + 1 < ngroups) group(g + 1, res + 8);
    }
    if (m_xw && row < d.M) d.ss_out[static_cast<size_t>(row) * d.ss_parts + k.n] = ss_acc;
  } else if constexpr (EPI == CHAIN_SWIGLU) {
    uint4 h2[4];
    for (int g = 0; g < ngroups; ++g) {
      float v[64];
      load_acc(t_row, g, ngroups + g, v);
      add_partials(d, tile, row_in_tile, g, ngroups + g, v);
      uint4 h4[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = silu(scale * v[8 * q + e]) * (scale * v[32 + 8 * q + e]);
        h4[q].x = pack_bf16x2(h[0], h[1]);
        h4[q].y = pack_bf16x2(h[2], h[3]);
        h4[q].z = pack_bf16x2(h[4], h[5]);
        h4[q].w = pack_bf16x2(h[6], h[7]);
      }
      if ((g & 1) == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) h2[q] = h4[q];
      }
      if ((g & 1) == 1 || g == ngroups - 1) {
        st.acquire();
        if ((g & 1) == 1) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            st.put(q, h2[q]);
            st.put(4 + q, h4[q]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) st.put(q, h4[q]);
        }
        st.store(m_out, k.n * (d.bn / 2) + (g >> 1) * 64, box_y, d.M);
      }
    }
  } else {  // CHAIN_QKV_HEADS
    for (int g = 0; g < ngroups; ++g) {
      float v[64];
      load_acc(t_row, 2 * g, 2 * g + 1, v);
      add_partials(d, tile, row_in_tile, 2 * g, 2 * g + 1, v);
#pragma unroll
      for (int j = 0; j < 64; ++j) v[j] *= scale;
      if (g < 2) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x1 = v[j], x2 = v[32 + j];
          v[j] = x1 * rc[j] - x2 * rs[j];
          v[32 + j] = x2 * rc[j] + x1 * rs[j];
        }
      }
      st.acquire();
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint4 o;
        o.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        o.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        o.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        o.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        st.put(q, o);
      }
      st.store(m_out, g * d.D + k.n * 64, box_y, d.M);
    }
  }
  tc_fence_before_sync();
  mbar_arrive(tempty_acc);
  if (d.splits > 1 && et == 0) d.arrivals[tile] = 0;  // ready for the next launch
  // Completion: this warp's TMA stores have written global memory, then one release per tile on
  // the row tile's counter.
  if (lane == 0) {
    bulk_wait_all();
    fence_proxy_async_global();
  }
  __syncwarp();
  __threadfence();
  named_barrier_sync(1, 128);
  if (et == 0) {
    __threadfence();
    atomicAdd(d.done + k.m, 1);
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1) k_chain(const __grid_constant__ ChainParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + kRingMax;
  uint64_t* tfull = empty + kRingMax;
  uint64_t* tempty = tfull + 2;
  uint64_t* task_full = tempty + 2;
  uint64_t* task_empty = task_full + kTaskSlots;
  uint64_t* mma_done = task_empty + kTaskSlots;
  uint64_t* teardown = mma_done + 1;
  Task* tasks = reinterpret_cast<Task*>(teardown + 1);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tasks + kTaskSlots);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* ticket_ok = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRingMax; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    for (int s = 0; s < kTaskSlots; ++s) {
      mbar_init(&task_full[s], 1);
      mbar_init(&task_empty[s], 1 + 4);  // the MMA issuer and the four epilogue warps
    }
    mbar_init(mma_done, 1);
    mbar_init(teardown, kThreads / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kChainMaxMaps; ++i)
      if (i < p.n_maps) tma_prefetch_desc(&p.maps[i]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 2 * kAccCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  if (threadIdx.x == 0) launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ tickets + TMA producer
    if (lane == 0) {
      grid_dependency_wait();  // earlier kernels of the stream (their outputs are the first operands)
      // Operand ring: ring_slots slots of slot_bytes (chosen per launch for its largest stage);
      // stage i uses slot i % ring_slots.
      const int n_ring = p.ring_slots;
      int sseq = 0;
      bool ok = true;
      auto alloc = [&](uint32_t) -> int {
        const int slot = sseq % n_ring;
        if (sseq >= n_ring &&
            !mbar_wait(&empty[slot], static_cast<uint32_t>(sseq / n_ring - 1) & 1u, abort_flag, p.err,
                       kErrTimeoutProducer))
          return -1;
        ++sseq;
        return slot;
      };
      for (int seq = 0; ok; ++seq) {
        const int slot = seq % kTaskSlots;
        const uint32_t tph = static_cast<uint32_t>(seq / kTaskSlots) & 1u;
        // Take the next ticket only once the accumulator buffer that task will use is free (the
        // epilogue of task seq - 2 is done): at most two tasks are bound to this CTA at a time,
        // so tickets go to CTAs that can start them soon.
        if (seq >= 2 && !mbar_wait(&tempty[seq & 1], ((seq >> 1) & 1) ^ 1, abort_flag, p.err, kErrTimeoutProducer)) {
          ok = false;
          break;
        }
        Task k;
        const int t = atomicAdd(p.ticket, 1);
        if (t >= p.total_tasks) {
          k = Task{0, 0, 0, 0, 0, 0, 1, 0};
        } else {
          decode(p, t, k);
        }
        if (seq >= kTaskSlots && !mbar_wait(&task_empty[slot], tph ^ 1, abort_flag, p.err, kErrTimeoutProducer)) {
          ok = false;
          break;
        }
        if (k.done) {
          tasks[slot] = k;
          mbar_arrive(&task_full[slot]);
          break;
        }
        const ChainStage& d = p.st[k.stage];
        const CUtensorMap* ma = &p.maps[d.map_a];
        const CUtensorMap* mb = &p.maps[d.map_b];
        const CUtensorMap* mb2 = d.map_b2 >= 0 ? &p.maps[d.map_b2] : mb;
        const uint32_t stage_bytes = static_cast<uint32_t>(kABytes + d.bn * 128);
        auto load_b = [&](int rs, int kb) {
          uint8_t* sb = smem + rs * p.slot_bytes + kABytes;
          if (d.epi == CHAIN_SWIGLU) {
            tma_load_2d(sb, mb, &full[rs], kb * BK, k.n * (d.bn / 2));
            tma_load_2d(sb + (d.bn / 2) * 128, mb2, &full[rs], kb * BK, k.n * (d.bn / 2));
          } else if (d.epi == CHAIN_QKV_HEADS) {
            // q, k and v rows of head n: three 64-row boxes of wqkv
            tma_load_2d(sb, mb, &full[rs], kb * BK, k.n * 64);
            tma_load_2d(sb + 64 * 128, mb, &full[rs], kb * BK, d.D + k.n * 64);
            tma_load_2d(sb + 128 * 128, mb, &full[rs], kb * BK, 2 * d.D + k.n * 64);
          } else {
            tma_load_2d(sb, mb, &full[rs], kb * BK, k.n * d.bn);
          }
        };
        auto load_a = [&](int rs, int kb) { tma_load_2d(smem + rs * p.slot_bytes, ma, &full[rs], kb * BK, k.m * BM); };
        // Weight tiles of the first stages: they depend on nothing.  The task is published (and
        // its stages consumed) only after its dependency wait, so these stages must fit in the
        // ring together: at most ring_slots of them.
        const int nkb = k.kb1 - k.kb0;
        const int pre = min(min(nkb, 4), n_ring);
        int pre_slot[4];
        for (int i = 0; i < pre && ok; ++i) {
          const int rs = alloc(stage_bytes);
          if (rs < 0) {
            ok = false;
            break;
          }
          pre_slot[i] = rs;
          mbar_arrive_expect_tx(&full[rs], stage_bytes);
          load_b(rs, k.kb0 + i);
        }
        // The activation rows: wait until the stage producing them has finished this row tile.
        if (ok && d.dep_stage >= 0) {
          ok = wait_counter_backoff(p.st[d.dep_stage].done + k.m, d.dep_target, abort_flag, p.err,
                                    kErrTimeoutProducer);
          fence_proxy_async_global();
        }
        if (!ok) {
          tasks[slot] = Task{0, 0, 0, 0, 0, 0, 1, 0};
          mbar_arrive(&task_full[slot]);
          break;
        }
        tasks[slot] = k;
        mbar_arrive(&task_full[slot]);
        for (int i = 0; i < pre; ++i) load_a(pre_slot[i], k.kb0 + i);
        for (int kb = k.kb0 + pre; kb < k.kb1; ++kb) {
          const int rs = alloc(stage_bytes);
          if (rs < 0) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[rs], stage_bytes);
          load_a(rs, kb);
          load_b(rs, kb);
        }
      }
      // Copies still in flight must land before the CTA may exit (error path; in the normal path
      // every issued stage has been consumed and these return at once).
      volatile int never = 0;
      for (int i = sseq > n_ring ? sseq - n_ring : 0; i < sseq; ++i)
        mbar_wait(&full[i % n_ring], static_cast<uint32_t>(i / n_ring) & 1u, &never, p.err, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int mseq = 0, acc = 0;  // stages consumed; accumulator buffer
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int seq = 0; ok; ++seq) {
        const int slot = seq % kTaskSlots;
        const uint32_t tph = static_cast<uint32_t>(seq / kTaskSlots) & 1u;
        if (!mbar_wait(&task_full[slot], tph, abort_flag, p.err, kErrTimeoutMma)) break;
        const Task k = tasks[slot];
        mbar_arrive(&task_empty[slot]);
        if (k.done) break;
        const ChainStage& d = p.st[k.stage];
        const uint32_t idesc = idesc_bf16(BM, d.bn, false);
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, kErrTimeoutMma)) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kAccCols);
        for (int kb = k.kb0; kb < k.kb1; ++kb) {
          const int rs = mseq % p.ring_slots;
          if (!mbar_wait(&full[rs], static_cast<uint32_t>(mseq / p.ring_slots) & 1u, abort_flag, p.err,
                         kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + rs * p.slot_bytes);
          const uint64_t adesc = sdesc_sw128(a_addr, 16, 1024);
          const uint64_t bdesc = sdesc_sw128(a_addr + kABytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb > k.kb0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[rs]);
          ++mseq;
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      umma_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, p.err, kErrTimeoutMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32)
    const int et = threadIdx.x - 64;
    Stager1 st{smem + OFF_STAGING + (warp - 2) * 4096, lane, 0};
    grid_dependency_wait();
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int seq = 0;; ++seq) {
      const int slot = seq % kTaskSlots;
      const uint32_t tph = static_cast<uint32_t>(seq / kTaskSlots) & 1u;
      const bool have = mbar_wait(&task_full[slot], tph, abort_flag, p.err, kErrTimeoutEpilogue);
      if (!named_barrier_and(2, 128, have)) break;
      const Task k = tasks[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&task_empty[slot]);
      if (k.done) break;
      const ChainStage& d = p.st[k.stage];
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(acc * kAccCols);
      bool ok;
      switch (d.epi) {
        case CHAIN_RESID:
          ok = epilogue_task<CHAIN_RESID>(p, d, k, t_row, &tfull[acc], &tempty[acc], acc_phase, quad, lane, et, st,
                                          abort_flag, ticket_ok);
          break;
        case CHAIN_SWIGLU:
          ok = epilogue_task<CHAIN_SWIGLU>(p, d, k, t_row, &tfull[acc], &tempty[acc], acc_phase, quad, lane, et, st,
                                           abort_flag, ticket_ok);
          break;
        default:
          ok = epilogue_task<CHAIN_QKV_HEADS>(p, d, k, t_row, &tfull[acc], &tempty[acc], acc_phase, quad, lane, et,
                                              st, abort_flag, ticket_ok);
          break;
      }
      if (!ok) break;
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // Teardown: TMEM is released only after every warp has finished with it (role code ran on
  // single lanes, so the warps meet on an mbarrier, one arrival per reconverged warp).
  tc_fence_before_sync();
  __syncwarp();
  if (lane == 0) mbar_arrive(teardown);
  {
    volatile int never = 0;
    mbar_wait(teardown, 0, &never, p.err, kErrTimeoutEpilogue);
  }
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

}  // namespace

int chain_ring_bytes() { return kRingBytes; }

cudaError_t launch_chain(const ChainParams& p, int grid, cudaStream_t s) {
  static unsigned long long attr_set_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(k_chain, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set_mask |= 1ull << dev;
  }
  if (p.total_tasks <= 0) return cudaSuccess;
  if (p.n_stages < 1 || p.n_stages > kChainMaxStages || p.n_maps > kChainMaxMaps || grid <= 0)
    return cudaErrorInvalidValue;
  if (p.ring_slots < 2 || p.ring_slots > kRingMax || p.slot_bytes % 1024 || p.ring_slots * p.slot_bytes > kRingBytes)
    return cudaErrorInvalidValue;

  for (int i = 0; i < p.n_stages; ++i) {
    const ChainStage& d = p.st[i];
    if (d.bn <= 0 || d.bn > kAccCols || d.bn % 64 || d.splits < 1 || d.splits > d.kb_total ||
        (d.epi == CHAIN_QKV_HEADS && d.bn != 192) || (d.epi == CHAIN_SWIGLU && d.bn % 128) ||
        d.dep_stage >= i || (d.splits > 1 && (!d.partials || !d.arrivals)) || !d.done ||
        kABytes + d.bn * 128 > p.slot_bytes)
      return cudaErrorInvalidValue;
  }
  return launch_pdl(k_chain, dim3(grid), dim3(kThreads), SMEM, s, p);
}

}  // namespace dsv4v
