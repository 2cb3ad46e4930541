// tcgen05 GEMM for the dense contractions of the vision block and the aligner:
//   wqkv (+ 2D rotary epilogue), output projection (+ residual), SwiGLU gate/up (+ silu*mul),
//   down projection (+ residual), aligner projection, patch embedding, PatchMerger projector.
//
// Structure (one persistent CTA per SM, 128 x BN output tiles, K in 64-element blocks):
//   warp 0      TMA producer: A and B tiles (128-byte swizzle) into a STAGES-deep smem ring
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer (M=128, N=BN, K=16 per instr.)
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (one TMEM lane = one output row
//               per thread), fused epilogue math, bf16 stores
//
// Work split (stream-K): the GEMM is U = tiles x (K / 64) units of one 64-deep K block of one
// output tile; CTA c of G owns units [c U / G, (c + 1) U / G), i.e. equal work per SM whatever
// the tile count.  A CTA walks its range as segments (a tile and a K-block range).  A segment
// that covers its whole tile is written directly.  A tile split between CTAs is finished by the
// CTA that owns its first K block: for that CTA the tile is the last segment of its range, while
// every other contributor meets the tile as its first segment, writes its fp32 partial to its
// scratch slot early and bumps the tile's counter.  The finisher waits (bounded) for the counter,
// adds the partials to its own accumulator in CTA order (deterministic) and runs the epilogue.
// Only finishers wait, and only on contributors that never wait, so the waits cannot cycle.
// The accumulator is double-buffered in TMEM so the epilogue of one segment overlaps the MMAs
// of the next.
#include <algorithm>
#include <unordered_map>

#include "common.cuh"
#include "internal.h"
#include "tile_util.cuh"

namespace dsv4v {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kMaxDynSmem = 232448;         // 227 KB per CTA
constexpr int kStagingBytes = 4 * 2 * 4096;  // per epilogue warp: two 32-row x 128-byte staging boxes
constexpr int kXwBytes = 256 * 4;            // the next norm's weights of a tile's columns

// PAIR: the CTA is one half of a CTA pair that computes a 256 x BN tile (tcgen05 cta_group::2):
// it holds 128 rows of A and BN / 2 rows of B per stage, and 128 x BN accumulators.
template <int BN, bool PAIR = false>
struct TileCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int RING_BUDGET = kMaxDynSmem - 1024 - 512 - kXwBytes - kStagingBytes;
  static constexpr int STAGES = RING_BUDGET / STAGE > 8 ? 8 : RING_BUDGET / STAGE;
  static constexpr int TMEM_COLS = (2 * BN <= 128) ? 128 : ((2 * BN <= 256) ? 256 : 512);
  static constexpr int OFF_STAGING = STAGES * STAGE;
  static constexpr int OFF_BARRIERS = OFF_STAGING + kStagingBytes;
  static constexpr int OFF_XW = OFF_BARRIERS + 512;
  static constexpr int SMEM = 1024 + OFF_XW + kXwBytes;
};

struct Params {
  int M, K, n_out;
  int tiles_m, kb_total;
  int owners;       // unit owners: CTAs, or CTA pairs
  long long units;  // tiles * kb_total
  __nv_bfloat16* out;
  int ldo;
  const __nv_bfloat16* resid;
  const float* cos;
  const float* sin;
  int rot_cols;
  float* partials;  // [G][BN / 4][128][4] fp32: a contributor's partial of a split tile
  int* counters;    // [tiles], zero between launches
  uint32_t* err;
  const float* norm_ss;  // folded RMSNorm, consumer side (see GemmArgs)
  int norm_parts, norm_stride;
  float norm_inv_d, norm_eps;
  __nv_bfloat16* xw_out;  // folded RMSNorm, producer side
  const float* xw_w;
  float* ss_out;
  int ss_parts;
  const float* bias;
  const void* l2_next[2];
  size_t l2_next_bytes[2];
  int b_early;
  int kb_split;  // MJ bit 2: K blocks of B read from tm_b; the rest from tm_b2
};

// ---------------------------------------------------------------------------- stream-K ranges
// Units are owned by CTAs, or by CTA pairs (owner c = CTAs 2c and 2c + 1).
__device__ __forceinline__ long long range_begin(const Params& p, int c) {
  return static_cast<long long>(c) * p.units / p.owners;
}
// Owner of unit u: the largest c with range_begin(c) <= u.
__device__ __forceinline__ int unit_owner(const Params& p, long long u) {
  return static_cast<int>(((u + 1) * p.owners - 1) / p.units);
}

struct Segment {
  int tile, m_tile, n_tile, kb0, kb1;
  bool first;  // first segment of this CTA's range
};

// Walks the segments of one owner's unit range.
struct SegmentWalker {
  long long u, u_end;
  bool first;
  __device__ __forceinline__ SegmentWalker(const Params& p, int owner) {
    u = range_begin(p, owner);
    u_end = range_begin(p, owner + 1);
    first = true;
  }
  __device__ __forceinline__ bool next(const Params& p, Segment& s) {
    if (u >= u_end) return false;
    s.tile = static_cast<int>(u / p.kb_total);
    s.kb0 = static_cast<int>(u - static_cast<long long>(s.tile) * p.kb_total);
    s.kb1 = static_cast<int>(min(static_cast<long long>(p.kb_total), s.kb0 + (u_end - u)));
    s.m_tile = s.tile % p.tiles_m;
    s.n_tile = s.tile / p.tiles_m;
    s.first = first;
    first = false;
    u += s.kb1 - s.kb0;
    return true;
  }
};



// Epilogue math of one 64-column accumulator group v[0..63] of output row `row`; the result
// goes to the warp's staging box (the caller stores it).  Pairs of columns use the packed fp32
// (f32x2) arithmetic.
//   STORE/RESID/QKV: v = accumulator columns [64g, 64g + 64) -> output columns n0 + 64g + j.
//     QKV: rot_c / rot_s hold the row's rotation table already multiplied by the folded-norm row
//     scale (pairs of columns, packed), so a rotated group needs no separate scaling.
//   SWIGLU: v[0..31] = gate columns, v[32..63] = up columns of output columns n0h + 32g + j;
//           written to chunks 4 (g & 1) .. 4 (g & 1) + 3 of the box.
//   RESID with the next norm prepared: the second box receives bf16(x * w_next).
template <int EPI, int BN, int NR>
__device__ __forceinline__ void epilogue_group(const Params& p, int row, int n_tile, int g, float (&v)[64],
                                               const uint64_t (&rot_c)[NR], const uint64_t (&rot_s)[NR],
                                               float row_scale, const uint4* resid, const float* xw_s, float& ss_acc,
                                               Stager& st, uint8_t* box, uint8_t* box2) {
  if (row >= p.M) return;
  const uint64_t rs2 = pk2(row_scale, row_scale);
  if constexpr (EPI == EPI_SWIGLU) {
    // silu(g r) (u r) with a = g r / 2: (a + a tanh(a)) (u r)
    const uint64_t hrs2 = pk2(0.5f * row_scale, 0.5f * row_scale);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float h[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const uint64_t a2 = mul2(pk2(v[8 * q + i], v[8 * q + i + 1]), hrs2);
        const uint64_t u2 = mul2(pk2(v[32 + 8 * q + i], v[32 + 8 * q + i + 1]), rs2);
        float a0, a1;
        upk2(a2, a0, a1);
        upk2(mul2(fma2(a2, pk2(tanh_approx(a0), tanh_approx(a1)), a2), u2), h[i], h[i + 1]);
      }
      uint4 o;
      o.x = pack_bf16x2(h[0], h[1]);
      o.y = pack_bf16x2(h[2], h[3]);
      o.z = pack_bf16x2(h[4], h[5]);
      o.w = pack_bf16x2(h[6], h[7]);
      st.put(box, 4 * (g & 1) + q, o);
    }
  } else {
    if constexpr (EPI == EPI_QKV_ROPE) {
      const int col = n_tile * BN + g * 64;
      if (col < p.rot_cols) {
        // (x1, x2) -> (x1 c - x2 s, x2 c + x1 s) for columns j and j + 32, two j at a time
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const uint64_t a = pk2(v[j], v[j + 1]), b = pk2(v[32 + j], v[33 + j]);
          const uint64_t c2 = rot_c[j >> 1], s2 = rot_s[j >> 1];
          upk2(sub2(mul2(a, c2), mul2(b, s2)), v[j], v[j + 1]);
          upk2(fma2(a, s2, mul2(b, c2)), v[32 + j], v[33 + j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 64; j += 2) upk2(mul2(pk2(v[j], v[j + 1]), rs2), v[j], v[j + 1]);
      }
    }
    if constexpr (EPI == EPI_GELU) {
      const float4* b4 = reinterpret_cast<const float4*>(p.bias + n_tile * BN + g * 64);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 bq = b4[q];
        v[4 * q] = gelu(v[4 * q] + bq.x);
        v[4 * q + 1] = gelu(v[4 * q + 1] + bq.y);
        v[4 * q + 2] = gelu(v[4 * q + 2] + bq.z);
        v[4 * q + 3] = gelu(v[4 * q + 3] + bq.w);
      }
    }
    if constexpr (EPI == EPI_STORE) {
      if (p.bias) {
        const float4* b4 = reinterpret_cast<const float4*>(p.bias + n_tile * BN + g * 64);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 bq = b4[q];
          upk2(add2(pk2(v[4 * q], v[4 * q + 1]), pk2(bq.x, bq.y)), v[4 * q], v[4 * q + 1]);
          upk2(add2(pk2(v[4 * q + 2], v[4 * q + 3]), pk2(bq.z, bq.w)), v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
    if constexpr (EPI == EPI_RESID) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint4 r = resid[q];
        upk2(add2(pk2(v[8 * q + 0], v[8 * q + 1]), bf16x2_f2(r.x)), v[8 * q + 0], v[8 * q + 1]);
        upk2(add2(pk2(v[8 * q + 2], v[8 * q + 3]), bf16x2_f2(r.y)), v[8 * q + 2], v[8 * q + 3]);
        upk2(add2(pk2(v[8 * q + 4], v[8 * q + 5]), bf16x2_f2(r.z)), v[8 * q + 4], v[8 * q + 5]);
        upk2(add2(pk2(v[8 * q + 6], v[8 * q + 7]), bf16x2_f2(r.w)), v[8 * q + 6], v[8 * q + 7]);
      }
    }
    uint4 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      o[q].x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
      o[q].y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
      o[q].z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
      o[q].w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
      st.put(box, q, o[q]);
    }
    if constexpr (EPI == EPI_RESID) {
      if (p.xw_out) {
        // Next RMSNorm's operand from the stored (bf16) x: bf16(x * w) and sum of x^2; w of the
        // tile's columns was staged in shared memory before the accumulator was ready.
        const float4* w4 = reinterpret_cast<const float4*>(xw_s + g * 64);
        uint64_t ss2 = 0ull;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 wa = w4[2 * q], wb = w4[2 * q + 1];
          const uint64_t x01 = bf16x2_f2(o[q].x), x23 = bf16x2_f2(o[q].y), x45 = bf16x2_f2(o[q].z),
                         x67 = bf16x2_f2(o[q].w);
          ss2 = fma2(x01, x01, ss2);
          ss2 = fma2(x23, x23, ss2);
          ss2 = fma2(x45, x45, ss2);
          ss2 = fma2(x67, x67, ss2);
          float t0, t1, t2, t3, t4, t5, t6, t7;
          upk2(mul2(x01, pk2(wa.x, wa.y)), t0, t1);
          upk2(mul2(x23, pk2(wa.z, wa.w)), t2, t3);
          upk2(mul2(x45, pk2(wb.x, wb.y)), t4, t5);
          upk2(mul2(x67, pk2(wb.z, wb.w)), t6, t7);
          uint4 t;
          t.x = pack_bf16x2(t0, t1);
          t.y = pack_bf16x2(t2, t3);
          t.z = pack_bf16x2(t4, t5);
          t.w = pack_bf16x2(t6, t7);
          st.put(box2, q, t);
        }
        float s0, s1;
        upk2(ss2, s0, s1);
        ss_acc += s0 + s1;
      }
    }
  }
}

// Folded-RMSNorm row scale of output row `row` (1 when the GEMM has no norm folded in).
__device__ __forceinline__ float norm_row_scale(const Params& p, int row) {
  if (!p.norm_ss) return 1.0f;
  const float* s = p.norm_ss + static_cast<size_t>(min(row, p.M - 1)) * p.norm_stride;
  float acc = 0.0f;
  for (int i = 0; i < p.norm_parts; ++i) acc += s[i];
  return 1.0f / sqrtf(acc * p.norm_inv_d + p.norm_eps);
}

// SwiGLU tiles of 352 columns: 176 gate + 176 up output columns, the gate half in TMEM columns
// [0, 176) and the up half in [192, 368) (two MMAs of N = 176 per K step, one tile per CTA).
template <int EPI, int BN>
constexpr bool kSwWide = EPI == EPI_SWIGLU && BN == 352;
// TMEM column of the up half of a SwiGLU accumulator.
template <int BN>
constexpr int kSwUp = BN == 352 ? 192 : BN / 2;

// Accumulator chunks (32 columns each) that make up epilogue group g.
template <int EPI, int BN>
__device__ __forceinline__ void group_chunks(int g, int& c0, int& c1) {
  if constexpr (EPI == EPI_SWIGLU) {
    c0 = g;
    c1 = kSwUp<BN> / 32 + g;
  } else {
    c0 = 2 * g;
    c1 = 2 * g + 1;
  }
}


// SwiGLU output columns [col0, col0 + n) of row `row` (n a multiple of 8) from group values v
// (gate in v[0..31], up in v[32..63]), straight to global memory: the tail of a 176-column tile,
// whose last 64-column box would spill into the next tile.
__device__ __forceinline__ void swiglu_store_direct(const Params& p, int row, int col0, float (&v)[64], float row_scale,
                                                    int n) {
  if (row >= p.M) return;
  __nv_bfloat16* dst = p.out + static_cast<size_t>(row) * p.ldo + col0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (8 * q >= n) break;
    float h[8];
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const uint64_t a2 = mul2(pk2(v[8 * q + i], v[8 * q + i + 1]), pk2(0.5f * row_scale, 0.5f * row_scale));
      const uint64_t u2 = mul2(pk2(v[32 + 8 * q + i], v[32 + 8 * q + i + 1]), pk2(row_scale, row_scale));
      float a0, a1;
      upk2(a2, a0, a1);
      upk2(mul2(fma2(a2, pk2(tanh_approx(a0), tanh_approx(a1)), a2), u2), h[i], h[i + 1]);
    }
    uint4 o;
    o.x = pack_bf16x2(h[0], h[1]);
    o.y = pack_bf16x2(h[2], h[3]);
    o.z = pack_bf16x2(h[4], h[5]);
    o.w = pack_bf16x2(h[6], h[7]);
    *reinterpret_cast<uint4*>(dst + 8 * q) = o;
  }
}

// Scratch slot of CTA c (a contributor writes at most one partial: its first segment).
// Layout [BN / 4][128 rows][4]: a warp's 32 rows of one 4-column group are 512 contiguous bytes.
template <int BN>
__device__ __forceinline__ float* partial_slot(const Params& p, int c) {
  return p.partials + static_cast<size_t>(c) * BM * BN;
}



// MJ: operand major-ness (see GemmArgs::mn_major).  An MN-major operand tile is loaded as
// 64 x 64 boxes of its stored [K, MN] matrix, one 128-byte-swizzled 8 KB atom column per 64
// MN indices, the atoms 8 KB apart (the descriptor's leading byte offset) and the 8-row K groups
// 1 KB apart (its stride byte offset); a K=16 step advances the start address by 2 KB.
template <int BN, int EPI, bool PAIR, int KS, int MJ = 0>
__global__ void __launch_bounds__(192, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
              const __grid_constant__ CUtensorMap tm_b2, const __grid_constant__ CUtensorMap tm_out,
              const __grid_constant__ CUtensorMap tm_xw, const Params p) {
  static_assert(KS == 1 || (!PAIR && (BN == 256 || (BN == 128 && KS == 2)) &&
                            (EPI == EPI_RESID || EPI == EPI_STORE || EPI == EPI_GELU)),
                "cluster split-K is built for 256-column (2 or 4 ranks) and 128-column (2 ranks) residual, "
                "store and GELU tiles");
  static_assert(MJ == 0 || (EPI == EPI_STORE && !PAIR && (KS == 1 || (MJ & 2) == 0) && BN % 64 == 0),
                "MN-major operands are built for STORE GEMMs without CTA pairs (with an MN-major A, "
                "without cluster split-K)");
  constexpr bool A_MN = (MJ & 2) != 0, B_MN = (MJ & 1) != 0, B_SPLIT = (MJ & 4) != 0;
  using C = TileCfg<BN, PAIR>;
  constexpr int BMT = PAIR ? 2 * BM : BM;  // rows of an output tile
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BARRIERS);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* teardown = mma_done + 1;  // one arrival per warp once its role is done
  uint64_t* xchg = teardown + 1;      // cluster split-K: the peers' partial slices have landed
  uint64_t* sent = xchg + 1;          // cluster split-K: every peer holds this CTA's slices
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sent + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* ticket = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // In a pair, rank 0 (the leader) issues the MMAs; its full and tempty barriers gather both
  // CTAs' loads and epilogue releases, the other barriers are signalled in both CTAs at once.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  // Cluster split-K (KS > 1): the KS CTAs of a cluster each run one K slice of the same tile and
  // then reduce-scatter the accumulator through distributed shared memory; rank kslice finishes
  // columns [kslice * BN / KS, (kslice + 1) * BN / KS).
  const uint32_t kslice = KS > 1 ? cluster_ctarank() : 0u;
  const int owner = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR ? 256 : 128);
    }
    mbar_init(mma_done, 1);
    mbar_init(teardown, blockDim.x / 32);
    mbar_init(xchg, 1);
    mbar_init(sent, KS > 1 ? KS - 1 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (EPI == EPI_SWIGLU || B_SPLIT) tma_prefetch_desc(&tm_b2);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();  // both CTAs' barriers are initialised before any remote use
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  if constexpr (PAIR) {
    // The leader's MMAs write the same TMEM columns in both CTAs.
    if (threadIdx.x == 0 &&
        ld_shared_cluster_u32(mapa_shared(smem_u32(const_cast<uint32_t*>(tmem_holder)), rank ^ 1u)) != tmem_base) {
      atomicCAS(p.err, 0u, static_cast<uint32_t>(kErrPairTmem));
      *abort_flag = 1;
    }
  }
  if (threadIdx.x == 0) launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_phase = 0;
      bool ok = true;
      // Stage s of both CTAs of a pair completes on the leader's full[s].
      const uint32_t full_leader = PAIR ? mapa_shared(smem_u32(full), 0) : 0u;
      const bool arrives = !PAIR || rank == 0;  // posts the expected bytes of the stage
      constexpr uint32_t kStageTx = PAIR ? 2 * C::STAGE : C::STAGE;
      auto load_a = [&](uint8_t* sa, int kb, int m_tile, int s) {
        if constexpr (A_MN) {
#pragma unroll
          for (int j = 0; j < BM / 64; ++j) tma_load_2d(sa + j * 8192, &tm_a, &full[s], m_tile * BM + 64 * j, kb * BK);
        } else if constexpr (PAIR)
          tma_load_2d_pair(sa, &tm_a, full_leader + 8u * s, kb * BK, m_tile * BMT + static_cast<int>(rank) * BM);
        else
          tma_load_2d(sa, &tm_a, &full[s], kb * BK, m_tile * BM);
      };
      auto load_b = [&](uint8_t* sb, int kb, int n_tile, int s) {
        if constexpr (B_MN) {
          const CUtensorMap* mb = &tm_b;
          int kr = kb;
          if (B_SPLIT && kb >= p.kb_split) {
            mb = &tm_b2;
            kr = kb - p.kb_split;
          }
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 8192, mb, &full[s], n_tile * BN + 64 * j, kr * BK);
        } else if constexpr (PAIR) {
          // The MMA's B is split along N: rank 0 holds rows [0, BN/2), rank 1 rows [BN/2, BN)
          // (SwiGLU: the gate rows and the up rows).
          if (EPI == EPI_SWIGLU)
            tma_load_2d_pair(sb, rank == 0 ? &tm_b : &tm_b2, full_leader + 8u * s, kb * BK, n_tile * (BN / 2));
          else
            tma_load_2d_pair(sb, &tm_b, full_leader + 8u * s, kb * BK, n_tile * BN + static_cast<int>(rank) * (BN / 2));
        } else if (EPI == EPI_SWIGLU) {
          tma_load_2d(sb, &tm_b, &full[s], kb * BK, n_tile * (BN / 2));
          tma_load_2d(sb + (BN / 2) * 128, &tm_b2, &full[s], kb * BK, n_tile * (BN / 2));
        } else {
          tma_load_2d(sb, &tm_b, &full[s], kb * BK, n_tile * BN);
        }
      };
      SegmentWalker walk(p, owner);
      Segment sg;
      // Weight tiles of the first stages do not depend on the previous kernel: start them before
      // waiting for it (b_early), then add the activation tiles.
      if (!p.b_early) grid_dependency_wait();
      int pre = 0;
      Segment first{};
      SegmentWalker peek = walk;
      if (peek.next(p, first)) {
        pre = min(STAGES, first.kb1 - first.kb0);
        for (int i = 0; i < pre; ++i) {
          if (arrives) mbar_arrive_expect_tx(&full[i], kStageTx);
          load_b(smem + i * C::STAGE + C::A_BYTES, first.kb0 + i, first.n_tile, i);
          issued |= 1u << i;
        }
      }
      grid_dependency_wait();
      for (int i = 0; i < pre; ++i) load_a(smem + i * C::STAGE, first.kb0 + i, first.m_tile, i);
      stage = pre % STAGES;
      phase = (pre == STAGES) ? 1u : 0u;
      while (ok && walk.next(p, sg)) {
        for (int kb = sg.first ? sg.kb0 + pre : sg.kb0; kb < sg.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, kErrTimeoutProducer)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE;
          if (arrives) mbar_arrive_expect_tx(&full[stage], kStageTx);
          load_a(sa, kb, sg.m_tile, stage);
          load_b(sa + C::A_BYTES, kb, sg.n_tile, stage);
          issued |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // The next GEMM's weights: this CTA's share into L2 while its own stages drain.
      if (ok) {
        for (int r = 0; r < 2; ++r) {
          if (!p.l2_next[r]) continue;
          const size_t share = (p.l2_next_bytes[r] + 16 * gridDim.x - 1) / (16 * gridDim.x) * 16;
          const size_t b0 = static_cast<size_t>(blockIdx.x) * share;
          const size_t b1 = min(p.l2_next_bytes[r], b0 + share);
          for (size_t o = b0; o < b1; o += 32768) {
            const size_t piece = b1 - o < 32768 ? b1 - o : 32768;
            prefetch_l2_bulk(static_cast<const uint8_t*>(p.l2_next[r]) + o, static_cast<uint32_t>(piece));
          }
        }
      }
      // Copies still in flight must land before the CTA may exit (error path only; in the
      // normal path every issued stage was consumed already and these return at once).  The
      // second CTA of a pair has no full barrier of its own: it waits until the MMAs released
      // each stage it filled.
      volatile int never = 0;
      for (int s = 0; s < STAGES; ++s) {
        if (!(issued & (1u << s))) continue;
        if (arrives) mbar_wait(&full[s], (issued_phase >> s) & 1u, &never, p.err, kErrTimeoutProducer);
        else mbar_wait(&empty[s], (issued_phase >> s) & 1u, &never, p.err, kErrTimeoutProducer);
      }
    }
    if constexpr (KS > 1) {
      __syncwarp();
      cluster_sync();  // the epilogue's cluster barrier
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (PAIR && rank != 0) {
      // The second CTA of a pair issues nothing; its TMEM is written by the leader's MMAs until
      // their final commit.
      if (lane == 0) {
        volatile int never = 0;
        mbar_wait(mma_done, 0, &never, p.err, kErrTimeoutMma);
      }
    } else if (lane == 0) {
      constexpr bool WIDE = kSwWide<EPI, BN>;
      constexpr uint32_t idesc = idesc_bf16_mn(BMT, WIDE ? BN / 2 : BN, A_MN, B_MN);
      // descriptor advance per K=16 step (address field in 16-byte units): 32 bytes inside a
      // K-major swizzle atom, two 8-row K groups (2 KB) for an MN-major tile
      constexpr uint64_t kStepA = A_MN ? 128 : 2, kStepB = B_MN ? 128 : 2;
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      SegmentWalker walk(p, owner);
      Segment sg;
      while (ok && walk.next(p, sg)) {
        const bool free_acc = PAIR ? mbar_wait_cluster(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, kErrTimeoutMma)
                                   : mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.err, kErrTimeoutMma);
        if (!free_acc) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(WIDE ? 0 : acc * BN);  // WIDE: one tile per CTA
        for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(smem + stage * C::STAGE);
          const uint32_t b_addr = a_addr + C::A_BYTES;
          const uint64_t adesc = sdesc_sw128(a_addr, A_MN ? 8192 : 16, 1024);
          const uint64_t bdesc = sdesc_sw128(b_addr, B_MN ? 8192 : 16, 1024);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            // +32 bytes per K=16 step inside the 128-byte swizzle atom (encoded >> 4).
            const uint32_t accum = (kb > sg.kb0 || k > 0) ? 1u : 0u;
            if constexpr (PAIR) {
              umma_bf16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
            } else if constexpr (WIDE) {
              // gate rows [0, BN / 2) of B, then up rows (1024-byte aligned: BN / 2 is a multiple of 8)
              const uint64_t bdesc_up = sdesc_sw128(b_addr + (BN / 2) * 128, 16, 1024);
              umma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, accum);
              umma_bf16(d_tmem + kSwUp<BN>, adesc + 2 * k, bdesc_up + 2 * k, idesc, accum);
            } else {
              umma_bf16(d_tmem, adesc + kStepA * k, bdesc + kStepB * k, idesc, accum);
            }
          }
          if constexpr (PAIR) umma_commit_pair(&empty[stage]);
          else umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if constexpr (PAIR) umma_commit_pair(&tfull[acc]);
        else umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // Every MMA issued so far completes before TMEM may be released.
      if constexpr (PAIR) umma_commit_pair(mma_done);
      else umma_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, p.err, kErrTimeoutMma);
    }
    __syncwarp();
    if constexpr (KS > 1) cluster_sync();  // the epilogue's cluster barrier (this CTA's MMAs are done)
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes [32 quad, 32 quad + 32) belong to this warp
    const int row_in_tile = quad * 32 + lane;
    const int et = threadIdx.x - 64;
    Stager st{smem + C::OFF_STAGING + (warp - 2) * 8192, lane, 0};
    // Hands an accumulator buffer back to the MMA issuer (the leader's barrier, in a pair).
    const uint32_t tempty_leader = PAIR ? mapa_shared(smem_u32(tempty), 0) : 0u;
    auto release_acc = [&](int buf) {
      if constexpr (PAIR) mbar_arrive_cluster(tempty_leader + 8u * static_cast<uint32_t>(buf));
      else mbar_arrive(&tempty[buf]);
    };
    constexpr int NGROUPS = BN / 64;
    int acc = 0;
    uint32_t acc_phase = 0;
    grid_dependency_wait();
    SegmentWalker walk(p, owner);
    Segment sg;
    if constexpr (KS > 1) {
      // ------------------------------------------------ cluster split-K: one K slice of one tile
      constexpr int GPR = NGROUPS / KS;  // 64-column groups finished by each rank
      constexpr int SLOT_BYTES = GPR * 16 * BM * 16;
      const int g0 = static_cast<int>(kslice) * GPR;
      const bool have = walk.next(p, sg);
      const int row = sg.m_tile * BM + row_in_tile;
      const int box_y = sg.m_tile * BM + quad * 32;
      // The folded-norm row scale, and the rotation table row pre-multiplied by it (packed pairs).
      float row_scale = norm_row_scale(p, row);
      pin(row_scale);
      uint64_t rot_c[EPI == EPI_QKV_ROPE ? 16 : 1], rot_s[EPI == EPI_QKV_ROPE ? 16 : 1];
      uint4 resid[EPI == EPI_RESID ? GPR * 8 : 1];
      if constexpr (EPI == EPI_QKV_ROPE) {
        const int prow = min(row, p.M - 1);
        const float4* c4 = reinterpret_cast<const float4*>(p.cos + static_cast<size_t>(prow) * 32);
        const float4* s4 = reinterpret_cast<const float4*>(p.sin + static_cast<size_t>(prow) * 32);
        const uint64_t rs2 = pk2(row_scale, row_scale);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 c = c4[q], sn = s4[q];
          rot_c[2 * q] = mul2(pk2(c.x, c.y), rs2);
          rot_c[2 * q + 1] = mul2(pk2(c.z, c.w), rs2);
          rot_s[2 * q] = mul2(pk2(sn.x, sn.y), rs2);
          rot_s[2 * q + 1] = mul2(pk2(sn.z, sn.w), rs2);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          pin(rot_c[j]);
          pin(rot_s[j]);
        }
      }
      if constexpr (EPI == EPI_RESID) {
        const uint4* r4 = reinterpret_cast<const uint4*>(p.resid + static_cast<size_t>(min(row, p.M - 1)) * p.ldo +
                                                         sg.n_tile * BN + g0 * 64);
#pragma unroll
        for (int q = 0; q < GPR * 8; ++q) resid[q] = r4[q];
#pragma unroll
        for (int q = 0; q < GPR * 8; ++q) pin(resid[q]);
      }
      float* xw_s = reinterpret_cast<float*>(smem + C::OFF_XW);
      if (EPI == EPI_RESID && p.xw_out && have)
        for (int i = et; i < BN; i += 128) xw_s[i] = p.xw_w[sg.n_tile * BN + i];
      float ss_acc = 0.0f;
      // The named barrier also publishes xw_s to the four epilogue warps.
      bool got = have && mbar_wait(&tfull[0], 0, abort_flag, p.err, kErrTimeoutEpilogue);
      got = named_barrier_and(2, 128, got);
      tc_fence_after_sync();
      // Reduce-scatter through the TMA rings, free once the MMAs are done.  Each CTA's ring holds
      // a receive area, one slot per sending rank, and a send area, one slice per peer, both in
      // the layout [group][16-byte column quad][row][4] (conflict-free for a warp's rows).  The
      // slices are staged locally, then moved by bulk copies that count on the peer's xchg.
      static_assert(2 * (KS - 1) * SLOT_BYTES <= STAGES * C::STAGE, "exchange areas exceed the ring");
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
      uint8_t* send = smem + (KS - 1) * SLOT_BYTES;
      if (got) {
#pragma unroll 1
        for (int j = 0; j < KS; ++j) {
          if (j == static_cast<int>(kslice)) continue;
          const int peer = j < static_cast<int>(kslice) ? j : j - 1;  // send slice of peer j
#pragma unroll 1
          for (int gi = 0; gi < GPR; ++gi) {
            int c0, c1;
            group_chunks<EPI, BN>(j * GPR + gi, c0, c1);
            uint32_t r0[32], r1[32];
            tmem_ld32(t_row + c0 * 32, r0);
            tmem_ld32(t_row + c1 * 32, r1);
            tmem_ld_wait(r0);
            tmem_ld_wait(r1);
            uint8_t* dst = send + peer * SLOT_BYTES + gi * 16 * BM * 16 + row_in_tile * 16;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              *reinterpret_cast<float4*>(dst + q * (BM * 16)) =
                  make_float4(__uint_as_float(r0[4 * q]), __uint_as_float(r0[4 * q + 1]),
                              __uint_as_float(r0[4 * q + 2]), __uint_as_float(r0[4 * q + 3]));
              *reinterpret_cast<float4*>(dst + (8 + q) * (BM * 16)) =
                  make_float4(__uint_as_float(r1[4 * q]), __uint_as_float(r1[4 * q + 1]),
                              __uint_as_float(r1[4 * q + 2]), __uint_as_float(r1[4 * q + 3]));
            }
          }
        }
      }
      fence_proxy_async_smem();  // the staged slices are read by the bulk-copy (async) proxy
      // Barrier 1: every CTA of the cluster has finished its MMAs (its receive area is free) and
      // staged its send slices.
      cluster_sync();
      if (et == 0) {
        if (have) mbar_arrive_expect_tx(xchg, (KS - 1) * SLOT_BYTES);
        if (got) {
          for (int j = 0; j < KS; ++j) {
            if (j == static_cast<int>(kslice)) continue;
            const int peer = j < static_cast<int>(kslice) ? j : j - 1;
            const int slot = static_cast<int>(kslice) < j ? static_cast<int>(kslice) : static_cast<int>(kslice) - 1;
            bulk_copy_to_peer(mapa_shared(smem_u32(smem + slot * SLOT_BYTES), static_cast<uint32_t>(j)),
                              send + peer * SLOT_BYTES, SLOT_BYTES, mapa_shared(smem_u32(xchg), static_cast<uint32_t>(j)));
          }
        }
      }
      // Every peer sends its slices whenever it has a tile (the cluster shares one tile).
      got = got && mbar_wait(xchg, 0, abort_flag, p.err, kErrTimeoutEpilogue);
      got = named_barrier_and(2, 128, got);
      // Every slice from a peer has landed, so its bulk copy no longer reads the peer's send
      // area: tell that peer.
      if (et == 0 && got)
        for (int j = 0; j < KS; ++j)
          if (j != static_cast<int>(kslice)) mbar_arrive_cluster(mapa_shared(smem_u32(sent), static_cast<uint32_t>(j)));
      if (got) {
        uint8_t* box = nullptr;
#pragma unroll
        for (int gi = 0; gi < GPR; ++gi) {
          const int g = g0 + gi;
          int c0, c1;
          group_chunks<EPI, BN>(g, c0, c1);
          float v[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = 0.0f;
          // Sum the K slices in rank order (deterministic).
#pragma unroll 1
          for (int src = 0; src < KS; ++src) {
            if (src == static_cast<int>(kslice)) {
              uint32_t r0[32], r1[32];
              tmem_ld32(t_row + c0 * 32, r0);
              tmem_ld32(t_row + c1 * 32, r1);
              tmem_ld_wait(r0);
              tmem_ld_wait(r1);
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                v[j] += __uint_as_float(r0[j]);
                v[32 + j] += __uint_as_float(r1[j]);
              }
            } else {
              const int slot = src < static_cast<int>(kslice) ? src : src - 1;
              const uint8_t* src_buf = smem + slot * SLOT_BYTES + gi * 16 * BM * 16 + row_in_tile * 16;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 lo = *reinterpret_cast<const float4*>(src_buf + q * (BM * 16));
                const float4 hi = *reinterpret_cast<const float4*>(src_buf + (8 + q) * (BM * 16));
                v[4 * q] += lo.x; v[4 * q + 1] += lo.y; v[4 * q + 2] += lo.z; v[4 * q + 3] += lo.w;
                v[32 + 4 * q] += hi.x; v[32 + 4 * q + 1] += hi.y; v[32 + 4 * q + 2] += hi.z; v[32 + 4 * q + 3] += hi.w;
              }
            }
          }
          uint8_t* box2 = nullptr;
          if (EPI == EPI_RESID && p.xw_out) st.acquire_both(box, box2);
          else box = st.acquire();
          epilogue_group<EPI, BN>(p, row, sg.n_tile, g, v, rot_c, rot_s, row_scale,
                                  EPI == EPI_RESID ? resid + (EPI == EPI_RESID ? gi * 8 : 0) : nullptr, xw_s, ss_acc,
                                  st, box, box2);
          st.store(box, &tm_out, sg.n_tile * BN + g * 64, box_y, p.M);
          if (EPI == EPI_RESID && p.xw_out) st.store(box2, &tm_xw, sg.n_tile * BN + g * 64, box_y, p.M);
        }
        if (EPI == EPI_RESID && p.xw_out && row < p.M)
          p.ss_out[static_cast<size_t>(row) * p.ss_parts + sg.n_tile * KS + static_cast<int>(kslice)] = ss_acc;
      }
      // No CTA leaves while a peer's bulk copy may still read its send area (bounded wait: a
      // peer that gave up never arrives).
      if (et == 0) {
        volatile int never = 0;
        mbar_wait_cluster(sent, 0, &never, p.err, kErrTimeoutEpilogue);
      }
    }
    bool xw_loaded = false;
    while (KS == 1 && walk.next(p, sg)) {
      const int row0 = sg.m_tile * BMT + static_cast<int>(rank) * BM;  // this CTA's rows of the tile
      const int row = row0 + row_in_tile;
      const int box_y = row0 + quad * 32;
      const int ctr = PAIR ? 2 * sg.tile + static_cast<int>(rank) : sg.tile;  // split-tile counter
      const bool finisher_or_full =
          (sg.kb0 == 0 && sg.kb1 == p.kb_total) ||
          owner == unit_owner(p, static_cast<long long>(sg.tile) * p.kb_total);
      // Inputs of the epilogue math fetched while the MMAs run: the rotation table row and the
      // residual row of this thread's output row, and the folded-norm row scale.
      // The folded-norm row scale, and the rotation table row pre-multiplied by it (packed pairs).
      float row_scale = norm_row_scale(p, row);
      pin(row_scale);
      uint64_t rot_c[EPI == EPI_QKV_ROPE ? 16 : 1], rot_s[EPI == EPI_QKV_ROPE ? 16 : 1];
      // The residual epilogue keeps RG groups (64 columns each) of the residual row in
      // registers and refills a slot RG groups ahead once its group is done.
      constexpr int RG = NGROUPS < 2 ? NGROUPS : 2;
      uint4 resid[EPI == EPI_RESID ? RG * 8 : 1];
      if constexpr (EPI == EPI_QKV_ROPE) {
        const int prow = min(row, p.M - 1);
        const float4* c4 = reinterpret_cast<const float4*>(p.cos + static_cast<size_t>(prow) * 32);
        const float4* s4 = reinterpret_cast<const float4*>(p.sin + static_cast<size_t>(prow) * 32);
        const uint64_t rs2 = pk2(row_scale, row_scale);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 c = c4[q], sn = s4[q];
          rot_c[2 * q] = mul2(pk2(c.x, c.y), rs2);
          rot_c[2 * q + 1] = mul2(pk2(c.z, c.w), rs2);
          rot_s[2 * q] = mul2(pk2(sn.x, sn.y), rs2);
          rot_s[2 * q + 1] = mul2(pk2(sn.z, sn.w), rs2);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          pin(rot_c[j]);
          pin(rot_s[j]);
        }
      }
      if constexpr (EPI == EPI_RESID) {
        if (finisher_or_full) {
          const uint4* r4 =
              reinterpret_cast<const uint4*>(p.resid + static_cast<size_t>(min(row, p.M - 1)) * p.ldo + sg.n_tile * BN);
#pragma unroll
          for (int q = 0; q < RG * 8; ++q) resid[q] = r4[q];
#pragma unroll
          for (int q = 0; q < RG * 8; ++q) pin(resid[q]);
        }
      }
      float* xw_s = reinterpret_cast<float*>(smem + C::OFF_XW);
      if (EPI == EPI_RESID && p.xw_out && finisher_or_full) {
        // After the first tile, every warp must be done with the previous tile's weights.
        if (xw_loaded) named_barrier_sync(3, 128);
        for (int i = et; i < BN; i += 128) xw_s[i] = p.xw_w[sg.n_tile * BN + i];
        xw_loaded = true;
      }
      float ss_acc = 0.0f;
      const bool got = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, kErrTimeoutEpilogue);
      // All four epilogue warps continue or stop together (TMEM loads are warp-collective and
      // the partial-tile path uses a named barrier); the barrier also publishes xw_s.
      if (!named_barrier_and(2, 128, got)) break;
      tc_fence_after_sync();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(kSwWide<EPI, BN> ? 0 : acc * BN);
      if (!finisher_or_full) {
        // Contributor to a tile finished by another CTA: park the partial, release it, move on.
        float* slot = partial_slot<BN>(p, blockIdx.x);
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_row + c * 32, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4*>(slot + ((c * 8 + q) * BM + row_in_tile) * 4) =
                make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                            __uint_as_float(r[4 * q + 3]));
        }
        tc_fence_before_sync();
        release_acc(acc);
        __threadfence();
        named_barrier_sync(1, 128);
        if (et == 0) atomicAdd(&p.counters[ctr], 1);
      } else {
        // Whole tile, or finisher of a split tile: wait for the other contributors (if any),
        // add their partials in CTA order, run the epilogue math, stage and store.
        const bool split = !(sg.kb0 == 0 && sg.kb1 == p.kb_total);
        int c_first = 0, c_last = 0;
        if (split) {
          const long long u_first = static_cast<long long>(sg.tile) * p.kb_total;
          c_first = unit_owner(p, u_first);
          c_last = unit_owner(p, u_first + p.kb_total - 1);
          if (et == 0) *ticket = wait_counter(&p.counters[ctr], c_last - c_first, abort_flag, p.err) ? 1 : 0;
          named_barrier_sync(1, 128);
          if (!*ticket) {
            tc_fence_before_sync();
            release_acc(acc);
            break;
          }
          __threadfence();
        }
        uint8_t* box = nullptr;
        constexpr bool WIDE = kSwWide<EPI, BN>;
        if constexpr (WIDE) {
          // 5.5 groups of 32 output columns, two at a time (one 64-column box): both groups'
          // accumulator columns are loaded together and their math is independent, so it can
          // interleave.  Columns [128, 176) are stored directly (a 64-column box would spill
          // into the next tile).
#pragma unroll 1
          for (int g = 0; g < 6; g += 2) {
            int c0, c1, c2, c3;
            group_chunks<EPI, BN>(g, c0, c1);
            group_chunks<EPI, BN>(g + 1, c2, c3);
            uint32_t r0[32], r1[32], r2[32], r3[32];
            tmem_ld32(t_row + c0 * 32, r0);
            tmem_ld32(t_row + c1 * 32, r1);
            tmem_ld32(t_row + c2 * 32, r2);
            tmem_ld32(t_row + c3 * 32, r3);
            tmem_ld_wait(r0);
            tmem_ld_wait(r1);
            tmem_ld_wait(r2);
            tmem_ld_wait(r3);
            float v[64], w[64];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              v[j] = __uint_as_float(r0[j]);
              v[32 + j] = __uint_as_float(r1[j]);
              w[j] = __uint_as_float(r2[j]);
              w[32 + j] = __uint_as_float(r3[j]);
            }
            const int col = sg.n_tile * (BN / 2) + 32 * g;
            if (g == 4) {
              swiglu_store_direct(p, row, col, v, row_scale, 32);
              swiglu_store_direct(p, row, col + 32, w, row_scale, 16);
              continue;
            }
            uint8_t* box2 = nullptr;
            box = st.acquire();
            epilogue_group<EPI, BN>(p, row, sg.n_tile, g, v, rot_c, rot_s, row_scale, nullptr, xw_s, ss_acc, st, box,
                                    box2);
            epilogue_group<EPI, BN>(p, row, sg.n_tile, g + 1, w, rot_c, rot_s, row_scale, nullptr, xw_s, ss_acc, st,
                                    box, box2);
            st.store(box, &tm_out, col, box_y, p.M);
          }
        }
        constexpr int NG = WIDE ? 0 : NGROUPS;
        // Unrolled for the residual epilogue so that its prefetched residual row stays in registers.
#pragma unroll(EPI == EPI_RESID ? NGROUPS : 1)
        for (int g = 0; g < NG; ++g) {
          int c0, c1;
          group_chunks<EPI, BN>(g, c0, c1);
          uint32_t r0[32], r1[32];
          tmem_ld32(t_row + c0 * 32, r0);
          tmem_ld32(t_row + c1 * 32, r1);
          tmem_ld_wait(r0);
          tmem_ld_wait(r1);
          float v[64];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] = __uint_as_float(r0[j]);
            v[32 + j] = __uint_as_float(r1[j]);
          }

          if (!WIDE && split) {  // WIDE plans give every CTA one whole tile
#pragma unroll 2
            for (int cc = c_first + 1; cc <= c_last; ++cc) {
              const float* src = partial_slot<BN>(p, PAIR ? 2 * cc + static_cast<int>(rank) : cc);
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
          uint8_t* box2 = nullptr;
          if (EPI == EPI_RESID && p.xw_out) st.acquire_both(box, box2);
          else if (EPI != EPI_SWIGLU || (g & 1) == 0) box = st.acquire();
          epilogue_group<EPI, BN>(p, row, sg.n_tile, g, v, rot_c, rot_s, row_scale,
                                  EPI == EPI_RESID ? resid + (EPI == EPI_RESID ? (g % RG) * 8 : 0) : nullptr, xw_s,
                                  ss_acc, st, box, box2);
          if constexpr (EPI == EPI_RESID) {
            if (g + RG < NGROUPS) {
              const uint4* r4 = reinterpret_cast<const uint4*>(
                  p.resid + static_cast<size_t>(min(row, p.M - 1)) * p.ldo + sg.n_tile * BN + (g + RG) * 64);
#pragma unroll
              for (int q = 0; q < 8; ++q) resid[(g % RG) * 8 + q] = r4[q];
            }
          }
          if constexpr (EPI == EPI_SWIGLU) {
            if ((g & 1) == 1 || g == NGROUPS - 1) st.store(box, &tm_out, sg.n_tile * (BN / 2) + (g >> 1) * 64, box_y, p.M);
          } else {
            st.store(box, &tm_out, sg.n_tile * BN + g * 64, box_y, p.M);
            if (EPI == EPI_RESID && p.xw_out) st.store(box2, &tm_xw, sg.n_tile * BN + g * 64, box_y, p.M);
          }
        }
        tc_fence_before_sync();
        release_acc(acc);
        if (EPI == EPI_RESID && p.xw_out && row < p.M)
          p.ss_out[static_cast<size_t>(row) * p.ss_parts + sg.n_tile] = ss_acc;
        if (split && et == 0) p.counters[ctr] = 0;  // ready for the next launch
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    st.drain();
  }

  // Teardown: TMEM is released only after every warp has finished with it.  Role code ran on
  // single lanes, so the warps meet on an mbarrier (one arrival per reconverged warp) rather than
  // on a CTA-wide bar.sync.
  tc_fence_before_sync();
  __syncwarp();
  if (lane == 0) mbar_arrive(teardown);
  {
    volatile int never = 0;
    mbar_wait(teardown, 0, &never, p.err, kErrTimeoutEpilogue);
  }
  // Neither CTA of a pair leaves (or frees TMEM) while the other may still signal its barriers.
  if constexpr (PAIR) cluster_sync();
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int BN, int EPI, bool PAIR = false, int KS = 1, int MJ = 0>
cudaError_t launch_one(const GemmPlan& plan, const GemmArgs& a, cudaStream_t s) {
  using C = TileCfg<BN, PAIR>;
  static unsigned long long attr_set_mask = 0;  // one bit per device, per instantiation
  auto kern = k_gemm_tc<BN, EPI, PAIR, KS, MJ>;
  if (PAIR && (plan.grid & 1)) return cudaErrorInvalidValue;
  if (kSwWide<EPI, BN> && (plan.grid != plan.work || plan.splits != 1 || a.n_out % (BN / 2)))
    return cudaErrorInvalidValue;  // one whole tile per CTA (a single accumulator)
  if (KS > 1 && (plan.grid % KS || plan.kb_total % KS || plan.grid != plan.work * KS)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set_mask |= 1ull << dev;
  }
  Params p;
  p.M = a.M;
  p.K = a.K;
  p.n_out = a.n_out;
  p.tiles_m = plan.tiles_m;
  p.kb_total = plan.kb_total;
  p.owners = PAIR ? plan.grid / 2 : plan.grid;
  p.units = static_cast<long long>(plan.tiles_m) * plan.tiles_n * plan.kb_total;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.ldo = a.ldo;
  p.resid = static_cast<const __nv_bfloat16*>(a.resid);
  p.cos = a.cos;
  p.sin = a.sin;
  p.rot_cols = a.rot_cols;
  p.partials = a.partials;
  p.counters = a.counters;
  p.err = a.err;
  p.norm_ss = a.norm_ss;
  p.norm_parts = a.norm_parts;
  p.norm_stride = a.norm_stride;
  p.norm_inv_d = a.norm_inv_d;
  p.norm_eps = a.norm_eps;
  p.xw_out = static_cast<__nv_bfloat16*>(a.xw_out);
  p.xw_w = a.xw_w;
  p.ss_out = a.ss_out;
  p.ss_parts = a.ss_parts;
  p.bias = a.bias;
  p.b_early = a.b_early ? 1 : 0;
  p.kb_split = a.kb_split;
  if ((MJ & 4) && (a.kb_split <= 0 || a.kb_split >= plan.kb_total || !a.tm_b2)) return cudaErrorInvalidValue;
  for (int r = 0; r < 2; ++r) {
    p.l2_next[r] = a.l2_next[r];
    p.l2_next_bytes[r] = a.l2_next_bytes[r];
    if (a.l2_next[r] && ((reinterpret_cast<uintptr_t>(a.l2_next[r]) & 15u) || (a.l2_next_bytes[r] & 15u)))
      return cudaErrorInvalidValue;
  }
  const CUtensorMap& ta = *a.tm_a;
  const CUtensorMap& tb2 = (EPI == EPI_SWIGLU || (MJ & 4)) ? *a.tm_b2 : *a.tm_b;
  const CUtensorMap& txw = a.tm_xw ? *a.tm_xw : *a.tm_out;
  if constexpr (PAIR || KS > 1)
    return launch_pdl_cluster(kern, dim3(plan.grid), dim3(192), C::SMEM, s, PAIR ? 2u : static_cast<unsigned>(KS), ta,
                              *a.tm_b, tb2, *a.tm_out, txw, p);
  else
    return launch_pdl(kern, dim3(plan.grid), dim3(192), C::SMEM, s, ta, *a.tm_b, tb2, *a.tm_out, txw, p);
}

// Tile widths each epilogue supports (the planner only picks these).
template <int EPI>
cudaError_t launch_bn(const GemmPlan& plan, const GemmArgs& a, cudaStream_t s) {
  if (plan.ks > 1) {
    // Cluster split-K: 256-column tiles over 2 or 4 ranks, 128-column tiles over 2.
    if constexpr (EPI == EPI_RESID || EPI == EPI_STORE || EPI == EPI_GELU) {
      if (plan.pair) return cudaErrorInvalidValue;
      if (plan.bn == 128 && plan.ks == 2) return launch_one<128, EPI, false, 2>(plan, a, s);
      if (plan.bn != 256) return cudaErrorInvalidValue;
      switch (plan.ks) {
        case 2: return launch_one<256, EPI, false, 2>(plan, a, s);
        case 4: return launch_one<256, EPI, false, 4>(plan, a, s);
        default: return cudaErrorInvalidValue;
      }
    }
    return cudaErrorInvalidValue;
  }
  if (plan.pair) {
    // CTA pairs: 256-row tiles.
    if constexpr (EPI == EPI_STORE || EPI == EPI_GELU) {
      return cudaErrorInvalidValue;
    } else if constexpr (EPI == EPI_SWIGLU) {
      if (plan.bn == 256) return launch_one<256, EPI, true>(plan, a, s);
      return cudaErrorInvalidValue;
    } else {
      switch (plan.bn) {
        case 128: return launch_one<128, EPI, true>(plan, a, s);
        case 256: return launch_one<256, EPI, true>(plan, a, s);
        default: return cudaErrorInvalidValue;
      }
    }
  }
  if constexpr (EPI == EPI_RESID) {
    switch (plan.bn) {
      case 64: return launch_one<64, EPI>(plan, a, s);
      case 128: return launch_one<128, EPI>(plan, a, s);
      case 256: return launch_one<256, EPI>(plan, a, s);
      default: return cudaErrorInvalidValue;
    }
  } else if constexpr (EPI == EPI_SWIGLU) {
    switch (plan.bn) {
      case 128: return launch_one<128, EPI>(plan, a, s);
      case 256: return launch_one<256, EPI>(plan, a, s);
      case 352: return launch_one<352, EPI>(plan, a, s);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (plan.bn) {
      case 64: return launch_one<64, EPI>(plan, a, s);
      case 128: return launch_one<128, EPI>(plan, a, s);
      case 192: return launch_one<192, EPI>(plan, a, s);
      case 256: return launch_one<256, EPI>(plan, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
}

// Cost model (cycles) of one SM's share of a GEMM, used to pick the tile width and the grid.
// Constants fitted to standalone, graph-replayed measurements on B200 (M = 784 and 3562, all four
// block GEMMs, every candidate tile width and grid):
//  - one 64-deep K block of a 128 x bn tile: ~600 cycles up to bn = 192 (the per-stage round trip
//    of TMA load, MMA and release, not the tensor pipe) and ~3.1 cycles per column above;
//  - a split tile: its partial (128 x bn fp32) written by each contributor and read back by the
//    finisher, the counter hand-off and the finisher's late epilogue, ~4000 + 40 bn cycles;
//  - per CTA: ~2000 cycles of set-up and first-load latency and ~12 cycles per output column.
double kblock_cycles(int bn) { return std::max(600.0, 3.1 * bn); }

double plan_cost(int bn, long long tiles, int kb_total, int grid, int* contrib_out) {
  const long long units = tiles * kb_total;
  const long long per_cta = (units + grid - 1) / grid;
  // Most contributors any tile has: ranges of per_cta units cut a tile of kb_total units.
  int contrib = 1;
  for (long long c = 0; c < grid; ++c) {
    const long long b = c * units / grid, e = (c + 1) * units / grid;
    if (b / kb_total != (e - 1) / kb_total || b % kb_total || e % kb_total) {
      const long long t = b / kb_total;
      const long long c0 = ((t * kb_total + 1) * grid - 1) / units;
      const long long c1 = (((t + 1) * kb_total) * grid - 1) / units;
      contrib = std::max<int>(contrib, static_cast<int>(c1 - c0 + 1));
    }
  }
  *contrib_out = contrib;
  double cost = per_cta * kblock_cycles(bn) + 2000.0 + 12.0 * bn;
  if (contrib > 1) cost += 4000.0 + 40.0 * bn;
  return cost;
}

// CTA pairs (256 x 256 tiles, tcgen05 cta_group::2, one tile's B split between two SMs) are
// taken when there are at least this many waves of pair tiles over the SM pairs.  Measured on
// B200 (standalone, graph-replayed): at M = 25000 pairs beat 128 x 256 single-CTA tiles by 1-7 %
// on all four GEMMs of the block (SwiGLU 235 -> 222 us, QKV 147 -> 137 us); at M = 3562 (1-4
// waves) they lose by 1-60 %, mostly to split-tile fix-ups.
constexpr int kPairMinWaves = 5;

// Cluster split-K costs: per 32 KB partial slice a CTA sends to a peer (staged in its ring, moved
// by a bulk DSMEM copy, summed by the peer; DSMEM moves ~30 B/ns per SM), and per CTA for the two
// cluster barriers and the staging.  Fitted on B200 at M = 784 (CUDA-graph step, 32 layers): the
// down projection (K = 2816) as 128-column tiles over 2 ranks beats 256-column tiles over 4 by
// 1.75 us per layer; the output projection (K = 1024) stays on 64-column single-CTA tiles
// (0.3 us per layer ahead of 128 x 2 ranks, 3.3 us ahead of 256 x 4).
constexpr double kExchangeCycles = 4200.0;
constexpr double kClusterCycles = 1000.0;

}  // namespace

GemmPlan plan_gemm_uncached(int epi, int M, int n_out, int K, int num_sms, size_t max_partial_bytes);

GemmPlan plan_gemm_whole(int M, int n_out, int K, int num_sms) {
  // Whole tiles per CTA only (the grid divides the tile count), 64-, 128- or 256-column tiles,
  // no cluster split-K: the plans that the MN-major STORE GEMMs are built for.
  GemmPlan best{};
  const int kb_total = (K + BK - 1) / BK;
  if (kb_total <= 0 || M <= 0 || num_sms <= 0) return best;
  const int tiles_m = (M + BM - 1) / BM;
  double best_cost = 1e300;
  for (int bn : {256, 128, 64}) {
    if (n_out % bn) continue;
    const long long tiles = static_cast<long long>(tiles_m) * (n_out / bn);
    for (long long g = std::min<long long>(num_sms, tiles); g >= 1; --g) {
      if (tiles % g) continue;
      int contrib = 1;
      const double cost = plan_cost(bn, tiles, kb_total, static_cast<int>(g), &contrib);
      if (contrib == 1 && cost < best_cost - 1e-9) {
        best_cost = cost;
        best.bn = bn;
        best.pair = 0;
        best.ks = 1;
        best.splits = 1;
        best.tiles_m = tiles_m;
        best.tiles_n = n_out / bn;
        best.kb_total = kb_total;
        best.work = static_cast<int>(tiles);
        best.grid = static_cast<int>(g);
        best.partial_bytes = 0;
        best.counters = 0;
      }
      break;  // the largest divisor that fits: more CTAs only add parallelism
    }
  }
  return best;
}

GemmPlan plan_gemm(int epi, int M, int n_out, int K, int num_sms, size_t max_partial_bytes) {
  // Plans depend only on the shape (and the scratch cap); each thread keeps the ones it has
  // computed.
  struct Key {
    int epi, M, n_out, K, sms;
    size_t cap;
    bool operator==(const Key& o) const {
      return epi == o.epi && M == o.M && n_out == o.n_out && K == o.K && sms == o.sms && cap == o.cap;
    }
  };
  struct KeyHash {
    size_t operator()(const Key& k) const {
      return ((((static_cast<size_t>(k.M) * 1000003u + k.n_out) * 1000003u + k.K) * 31u + k.epi) * 1009u + k.sms) *
                 131u +
             k.cap;
    }
  };
  thread_local std::unordered_map<Key, GemmPlan, KeyHash> cache;
  const Key key{epi, M, n_out, K, num_sms, max_partial_bytes};
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  if (cache.size() > 1024) cache.clear();
  GemmPlan best = plan_gemm_uncached(epi, M, n_out, K, num_sms, max_partial_bytes);
  cache[key] = best;
  return best;
}

GemmPlan plan_gemm_uncached(int epi, int M, int n_out, int K, int num_sms, size_t max_partial_bytes) {
  GemmPlan best{};
  const int kb_total = (K + BK - 1) / BK;  // a ragged last K block reads zeros past the end
  if (kb_total <= 0 || M <= 0 || num_sms <= 0) return best;
  // CTA pairs with 256-column tiles, stream-K over all SM pairs, when there is enough work.
  if ((epi == EPI_RESID || epi == EPI_QKV_ROPE || epi == EPI_SWIGLU) && n_out % (epi == EPI_SWIGLU ? 128 : 256) == 0) {
    const int tiles_m = (M + 2 * BM - 1) / (2 * BM);
    const int tiles_n = n_out / (epi == EPI_SWIGLU ? 128 : 256);
    const long long tiles = static_cast<long long>(tiles_m) * tiles_n;
    const int pairs = num_sms / 2;
    int contrib = 1;
    plan_cost(256, tiles, kb_total, pairs, &contrib);
    const size_t partial = contrib > 1 ? static_cast<size_t>(2 * pairs) * BM * 256 * sizeof(float) : 0;
    if (pairs > 0 && tiles >= static_cast<long long>(kPairMinWaves) * pairs && contrib <= 2 &&
        partial <= max_partial_bytes) {
      best.bn = 256;
      best.pair = 1;
      best.ks = 1;
      best.splits = contrib;
      best.tiles_m = tiles_m;
      best.tiles_n = tiles_n;
      best.kb_total = kb_total;
      best.work = static_cast<int>(tiles);
      best.grid = 2 * pairs;
      best.partial_bytes = partial;
      best.counters = contrib > 1 ? static_cast<int>(tiles) * 2 : 0;
      return best;
    }
  }
  double best_cost = 1e300;
  const int tiles_m = (M + BM - 1) / BM;
  // SwiGLU with few row tiles: 176 output columns per tile (two MMAs of N = 176 into 352
  // accumulator columns), one tile per CTA, when those tiles fit one wave and 128-column tiles
  // would not (M = 784: 112 CTAs instead of 154 tiles on 77 CTAs, two each).
  if (epi == EPI_SWIGLU && n_out % 176 == 0) {
    const long long wide = static_cast<long long>(tiles_m) * (n_out / 176);
    const long long narrow = static_cast<long long>(tiles_m) * ((n_out + 127) / 128);
    if (wide <= num_sms && narrow > num_sms) {
      best.bn = 352;
      best.pair = 0;
      best.ks = 1;
      best.splits = 1;
      best.tiles_m = tiles_m;
      best.tiles_n = n_out / 176;
      best.kb_total = kb_total;
      best.work = static_cast<int>(wide);
      best.grid = static_cast<int>(wide);
      best.partial_bytes = 0;
      best.counters = 0;
      return best;
    }
  }
  const int cands[4] = {256, 192, 128, 64};
  for (int bn : cands) {
    // Epilogue constraints: SwiGLU stores 64-column boxes of two 32-column groups (bn / 2 a
    // multiple of 64); the residual epilogue is built for bn in {64, 128, 256}.
    if (epi == EPI_SWIGLU && (bn / 2) % 64) continue;
    if (epi == EPI_RESID && bn == 192) continue;
    const int n_cols_per_tile = (epi == EPI_SWIGLU) ? bn / 2 : bn;
    if (n_out % n_cols_per_tile) continue;
    const int tiles_n = n_out / n_cols_per_tile;
    const long long tiles = static_cast<long long>(tiles_m) * tiles_n;
    const long long units = tiles * kb_total;
    // Grids: every SM; t whole tiles per CTA (t = 1..4); the largest divisor of the tile count
    // that fits the SMs (equal whole tiles per CTA); or s CTAs per tile (split-K by s).
    int grids[10];
    int n_grids = 0;
    grids[n_grids++] = static_cast<int>(std::min<long long>(num_sms, units));
    for (int t = 1; t <= 4; ++t) {
      const long long g = (tiles + t - 1) / t;
      if (g <= num_sms) grids[n_grids++] = static_cast<int>(g);
    }
    for (long long g = std::min<long long>(num_sms, tiles); g >= 1; --g)
      if (tiles % g == 0) {
        grids[n_grids++] = static_cast<int>(g);
        break;
      }
    for (int s = 2; s <= 4; ++s)
      if (tiles * s <= num_sms && tiles * s <= units) grids[n_grids++] = static_cast<int>(tiles * s);
    for (int gi = 0; gi < n_grids; ++gi) {
      int contrib = 1;
      const double cost = plan_cost(bn, tiles, kb_total, grids[gi], &contrib);
      if (contrib > 2) continue;  // more contributors leave straggling finishers (measured)
      const size_t partial = contrib > 1 ? static_cast<size_t>(grids[gi]) * BM * bn * sizeof(float) : 0;
      if (partial > max_partial_bytes) continue;
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best.bn = bn;
        best.pair = 0;
        best.ks = 1;
        best.splits = contrib;
        best.tiles_m = tiles_m;
        best.tiles_n = tiles_n;
        best.kb_total = kb_total;
        best.work = static_cast<int>(tiles);
        best.grid = grids[gi];
        best.partial_bytes = partial;
        best.counters = contrib > 1 ? static_cast<int>(tiles) : 0;
      }
    }
  }
  // Cluster split-K for residual, store and GELU tiles (256 columns over 2 or 4 ranks, 128 over
  // 2): full-rate MMAs even when there are too few tiles for the SMs, without the global-memory
  // split-tile fix-up.
  if (epi == EPI_RESID || epi == EPI_STORE || epi == EPI_GELU) {
    const int shapes[3][2] = {{256, 2}, {256, 4}, {128, 2}};
    for (const auto& sh : shapes) {
      const int bn = sh[0], ks = sh[1];
      if (n_out % bn) continue;
      const long long tiles = static_cast<long long>(tiles_m) * (n_out / bn);
      if (kb_total % ks || tiles * ks > num_sms) continue;
      const double slices = (ks - 1) * (static_cast<double>(BM) * (bn / ks) * 4.0) / 32768.0;
      const double cost = (kb_total / ks) * kblock_cycles(bn) + 2000.0 + 12.0 * (bn / ks) +
                          kExchangeCycles * slices + kClusterCycles;
      if (cost < best_cost - 1e-9) {
        best_cost = cost;
        best.bn = bn;
        best.pair = 0;
        best.ks = ks;
        best.splits = 1;
        best.tiles_m = tiles_m;
        best.tiles_n = n_out / bn;
        best.kb_total = kb_total;
        best.work = static_cast<int>(tiles);
        best.grid = static_cast<int>(tiles * ks);
        best.partial_bytes = 0;
        best.counters = 0;
      }
    }
  }
  return best;
}

// STORE GEMMs with MN-major operands (the backward's input and weight gradients): whole tiles
// per CTA, or cluster split-K when A is K-major.
template <int MJ>
cudaError_t launch_bn_mn(const GemmPlan& plan, const GemmArgs& a, cudaStream_t s) {
  if (plan.pair || plan.splits != 1) return cudaErrorInvalidValue;
  if (plan.ks > 1) {
    // cluster split-K (input gradients with a long K): B MN-major only
    if constexpr ((MJ & 2) == 0) {
      if (plan.bn == 128 && plan.ks == 2) return launch_one<128, EPI_STORE, false, 2, MJ>(plan, a, s);
      if (plan.bn == 256 && plan.ks == 2) return launch_one<256, EPI_STORE, false, 2, MJ>(plan, a, s);
      if (plan.bn == 256 && plan.ks == 4) return launch_one<256, EPI_STORE, false, 4, MJ>(plan, a, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (plan.bn) {
    case 64: return launch_one<64, EPI_STORE, false, 1, MJ>(plan, a, s);
    case 128: return launch_one<128, EPI_STORE, false, 1, MJ>(plan, a, s);
    case 256: return launch_one<256, EPI_STORE, false, 1, MJ>(plan, a, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm_tc(int epi, const GemmPlan& plan, const GemmArgs& a, cudaStream_t s) {
  if (a.mn_major != 0) {
    if (epi != EPI_STORE) return cudaErrorInvalidValue;
    switch (a.mn_major) {
      case 1: return launch_bn_mn<1>(plan, a, s);
      case 3: return launch_bn_mn<3>(plan, a, s);
      case 5: return launch_bn_mn<5>(plan, a, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (epi) {
    case EPI_STORE: return launch_bn<EPI_STORE>(plan, a, s);
    case EPI_RESID: return launch_bn<EPI_RESID>(plan, a, s);
    case EPI_QKV_ROPE: return launch_bn<EPI_QKV_ROPE>(plan, a, s);
    case EPI_SWIGLU: return launch_bn<EPI_SWIGLU>(plan, a, s);
    case EPI_GELU: return launch_bn<EPI_GELU>(plan, a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsv4v
