// Gradient of the varlen full attention on tcgen05 (head_dim 64), the chain rule of
// O = softmax(Q K^T / sqrt(hd)) V per image and head:
//   P = 2^(Q K^T c - lse)          c = log2(e) / sqrt(hd), lse from the forward kernel
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),  D = rowsum(dO * O)
//   dQ = dS K / sqrt(hd),  dK = dS^T Q / sqrt(hd)
// Two kernels, so that no output needs a reduction across CTAs (deterministic):
//   k_attn_bwd_kv  one CTA per (image, 128-key tile, head), looping over the image's query
//                  tiles: S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and dS^T (bf16) back into
//                  TMEM by the compute warps, then dV += P^T dO and dK += dS^T Q with the A
//                  operand read from TMEM; K and V stay in shared memory.
//   k_attn_bwd_q   one CTA per (image, 128-query tile, head), looping over key tiles:
//                  S = Q K^T, dP = dO V^T, dS = P * (dP - D) back into TMEM, dQ += dS K.
// Queries or keys past the end of the image get P = 0 (their lse is +inf, or the scores are
// masked), so rows that TMA reads from the next image contribute nothing.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2..5
// compute, one TMEM lane (one key row, resp. query row) per thread.
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

constexpr int HD = 64;
constexpr int TT = 128;                  // rows of a tile
constexpr int TILE = TT * HD * 2;        // 16 KB
constexpr int RING = 3;                  // streamed stages (two tiles each)
constexpr int OFF_RES = 0;               // two resident tiles
constexpr int OFF_RING = 2 * TILE;
constexpr int OFF_VEC = OFF_RING + RING * 2 * TILE;   // [RING][2][128] fp32: lse and D per query
constexpr int OFF_BAR = OFF_VEC + RING * 2 * TT * 4;
constexpr int SMEM_BYTES = 1024 + OFF_BAR + 512;
constexpr int kThreads = 192;
// TMEM columns
constexpr uint32_t T_S = 0, T_DP = 128, T_P = 256, T_DS = 320, T_ACC0 = 384, T_ACC1 = 448;

struct BwdParams {
  int n_heads, vision_dim;
  int64_t lse_ld;       // row stride of lse / rowdot ([n_heads, lse_ld])
  float c_log2;         // log2(e) / sqrt(hd)
  float scale;          // 1 / sqrt(hd)
  const float* lse;
  const float* rowdot;
  __nv_bfloat16* dqkv;  // [P, 3D]
  uint32_t* err;
};

__device__ __forceinline__ void find_tile(const AttnSchedule& s, int item, int& img, int& local) {
  int lo = 0, hi = s.n_images - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.item_start[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  img = lo;
  local = item - s.item_start[lo];
}

// One 128 x 128 x 64 product into TMEM: A and B both K-major [128 rows x 64] tiles in smem.
__device__ __forceinline__ void mma_tile_kmajor(uint32_t d, uint32_t a_addr, uint32_t b_addr) {
  constexpr uint32_t idesc = idesc_bf16(TT, TT, false);
  const uint64_t ad = sdesc_sw128(a_addr, 16, 1024), bd = sdesc_sw128(b_addr, 16, 1024);
#pragma unroll
  for (int k = 0; k < HD / 16; ++k) umma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, k > 0 ? 1u : 0u);
}

// acc (+)= A[tmem, 128 x 128 bf16] . B where B is the [128 rows (K) x 64 columns (N)] smem tile,
// N contiguous (MN-major).
__device__ __forceinline__ void mma_tmem_a(uint32_t d, uint32_t a_tmem, uint32_t b_addr, bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16(TT, HD, true);
#pragma unroll
  for (int kk = 0; kk < TT / 16; ++kk) {
    const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, TILE, 1024);
    umma_bf16_tmem_a(d, a_tmem + kk * 8, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Stores one 64-column fp32 accumulator row (scaled) as bf16 at dst (16-byte aligned).
__device__ __forceinline__ void store_row64(__nv_bfloat16* dst, const uint32_t* v, float scale) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint4 o;
    o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * scale, __uint_as_float(v[8 * q + 1]) * scale);
    o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * scale, __uint_as_float(v[8 * q + 3]) * scale);
    o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * scale, __uint_as_float(v[8 * q + 5]) * scale);
    o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * scale, __uint_as_float(v[8 * q + 7]) * scale);
    d4[q] = o;
  }
}

// KV: one CTA per (key tile, head): dK and dV.  !KV: one CTA per (query tile, head): dQ.
template <bool KV>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_bwd_tc(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ AttnSchedule sched, const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* res_full = bars;
  uint64_t* full = res_full + 1;
  uint64_t* empty = full + RING;
  uint64_t* sdp_full = empty + RING;
  uint64_t* s_free = sdp_full + 1;
  uint64_t* p_full = s_free + 1;
  uint64_t* pv_done = p_full + 1;
  uint64_t* mma_done = pv_done + 1;
  uint64_t* teardown = mma_done + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* vec = reinterpret_cast<float*>(smem + OFF_VEC);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int img, local;
  find_tile(sched, blockIdx.x, img, local);
  const int head = blockIdx.y;
  const int row0 = sched.img_row0[img];
  const int len = sched.img_len[img];
  const int n_t = (len + TT - 1) / TT;  // streamed tiles: query tiles (KV) or key tiles (!KV)
  const int tile_row = row0 + local * TT;  // first row of the resident tile
  const int D = p.vision_dim;
  const int col_q = head * HD, col_k = D + head * HD, col_v = 2 * D + head * HD;

  if (threadIdx.x == 0) {
    mbar_init(res_full, 1);
    for (int s = 0; s < RING; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(sdp_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    mbar_init(teardown, kThreads / 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_qkv);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  if (threadIdx.x == 0) launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      grid_dependency_wait();
      // Resident: K and V of this key tile (KV), or Q and dO of this query tile (!KV).
      mbar_arrive_expect_tx(res_full, 2 * TILE);
      if (KV) {
        tma_load_2d(smem + OFF_RES, &tm_qkv, res_full, col_k, tile_row);
        tma_load_2d(smem + OFF_RES + TILE, &tm_qkv, res_full, col_v, tile_row);
      } else {
        tma_load_2d(smem + OFF_RES, &tm_qkv, res_full, col_q, tile_row);
        tma_load_2d(smem + OFF_RES + TILE, &tm_do, res_full, head * HD, tile_row);
      }
      int issued = 0;
      for (int t = 0; t < n_t; ++t) {
        const int s = t % RING;
        if (!mbar_wait(&empty[s], ((t / RING) & 1) ^ 1, abort_flag, p.err, kErrTimeoutProducer)) break;
        mbar_arrive_expect_tx(&full[s], 2 * TILE);
        uint8_t* st = smem + OFF_RING + s * 2 * TILE;
        if (KV) {  // Q_t and dO_t
          tma_load_2d(st, &tm_qkv, &full[s], col_q, row0 + t * TT);
          tma_load_2d(st + TILE, &tm_do, &full[s], head * HD, row0 + t * TT);
        } else {   // K_t and V_t
          tma_load_2d(st, &tm_qkv, &full[s], col_k, row0 + t * TT);
          tma_load_2d(st + TILE, &tm_qkv, &full[s], col_v, row0 + t * TT);
        }
        issued = t + 1;
      }
      // Copies still in flight land before exit (returns at once in the normal path).
      volatile int never = 0;
      mbar_wait(res_full, 0, &never, p.err, kErrTimeoutProducer);
      for (int t = issued > RING ? issued - RING : 0; t < issued; ++t)
        mbar_wait(&full[t % RING], (t / RING) & 1, &never, p.err, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t res = smem_u32(smem + OFF_RES);
      // KV: S^T = K Q_t^T, dP^T = V dO_t^T.   !KV: S = Q K_t^T, dP = dO V_t^T.
      auto issue_sdp = [&](int t) {
        const uint32_t st = smem_u32(smem + OFF_RING + (t % RING) * 2 * TILE);
        mma_tile_kmajor(tmem_base + T_S, res, st);
        mma_tile_kmajor(tmem_base + T_DP, res + TILE, st + TILE);
        umma_commit(sdp_full);
      };
      // KV: dV += P^T dO_t, dK += dS^T Q_t.   !KV: dQ += dS K_t.
      auto issue_acc = [&](int t) {
        const uint32_t st = smem_u32(smem + OFF_RING + (t % RING) * 2 * TILE);
        if (KV) {
          mma_tmem_a(tmem_base + T_ACC0, tmem_base + T_P, st + TILE, t > 0);
          mma_tmem_a(tmem_base + T_ACC1, tmem_base + T_DS, st, t > 0);
        } else {
          mma_tmem_a(tmem_base + T_ACC0, tmem_base + T_DS, st, t > 0);
        }
        umma_commit(&empty[t % RING]);
        umma_commit(pv_done);
      };
      bool ok = mbar_wait(res_full, 0, abort_flag, p.err, kErrTimeoutMma);
      if (ok && n_t > 0) ok = mbar_wait(&full[0], 0, abort_flag, p.err, kErrTimeoutMma);
      if (ok && n_t > 0) {
        tc_fence_after_sync();
        issue_sdp(0);
      }
      for (int t = 0; t < n_t && ok; ++t) {
        if (t + 1 < n_t) {
          // S and dP of the next tile as soon as the compute warps have this one in registers.
          const int u = t + 1;
          ok = mbar_wait(&full[u % RING], (u / RING) & 1, abort_flag, p.err, kErrTimeoutMma) &&
               mbar_wait(s_free, t & 1, abort_flag, p.err, kErrTimeoutMma);
          if (!ok) break;
          tc_fence_after_sync();
          issue_sdp(u);
        }
        ok = mbar_wait(p_full, t & 1, abort_flag, p.err, kErrTimeoutMma);
        if (!ok) break;
        tc_fence_after_sync();
        issue_acc(t);
      }
      umma_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, p.err, kErrTimeoutMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ compute warps
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // TMEM lane = row of the resident tile
    const int et = threadIdx.x - 64;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    grid_dependency_wait();
    const float* lse_h = p.lse + static_cast<int64_t>(head) * p.lse_ld;
    const float* dot_h = p.rowdot + static_cast<int64_t>(head) * p.lse_ld;
    // !KV: this thread's query row has fixed lse and D.
    float my_lse = 0.0f, my_dot = 0.0f;
    const int my_row = local * TT + r;  // row of the resident tile inside the image
    if (!KV && my_row < len) {
      my_lse = lse_h[row0 + my_row];
      my_dot = dot_h[row0 + my_row];
    }
    // KV: lse and D of the streamed query tile t, one query per thread, staged in smem (prefetched
    // one tile ahead into registers).
    float nx_lse = INFINITY, nx_dot = 0.0f;
    if (KV && r < len) {
      nx_lse = lse_h[row0 + r];
      nx_dot = dot_h[row0 + r];
    }
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      if (KV) {
        float* vl = vec + (t % RING) * 2 * TT;
        vl[r] = nx_lse;
        vl[TT + r] = nx_dot;
        const int qn = (t + 1) * TT + r;
        nx_lse = INFINITY;
        nx_dot = 0.0f;
        if (t + 1 < n_t && qn < len) {
          nx_lse = lse_h[row0 + qn];
          nx_dot = dot_h[row0 + qn];
        }
        named_barrier_sync(1, 128);
      }
      const bool got = mbar_wait(sdp_full, t & 1, abort_flag, p.err, kErrTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      if (t > 0) {
        // P/dS of the previous tile are free once its accumulating products have completed.
        const bool done = mbar_wait(pv_done, (t - 1) & 1, abort_flag, p.err, kErrTimeoutEpilogue);
        if (!__all_sync(0xffffffffu, done)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
      }
      const float* vl = vec + (t % RING) * 2 * TT;
#pragma unroll 1
      for (int c = 0; c < TT / 32; ++c) {
        uint32_t sv[32], dpv[32];
        tmem_ld32(t_lane + T_S + c * 32, sv);
        tmem_ld32(t_lane + T_DP + c * 32, dpv);
        tmem_ld_wait(sv);
        tmem_ld_wait(dpv);
        if (c == TT / 32 - 1) {
          tc_fence_before_sync();
          mbar_arrive(s_free);  // S and dP are in registers: the next tile's products may land
        }
        uint32_t pp[16], ds[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float e[2], g[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = c * 32 + i + u;
            float lse, dot;
            if (KV) {
              lse = vl[col];  // column = query
              dot = vl[TT + col];
            } else {
              lse = my_lse;
              dot = my_dot;
            }
            float x = __uint_as_float(sv[i + u]) * p.c_log2 - lse;
            if (!KV && (t * TT + col >= len || my_row >= len)) x = -INFINITY;  // key past the image
            e[u] = ex2_approx(x);
            g[u] = e[u] * (__uint_as_float(dpv[i + u]) - dot);
          }
          pp[i >> 1] = pack_bf16x2(e[0], e[1]);
          ds[i >> 1] = pack_bf16x2(g[0], g[1]);
        }
        if (KV) tmem_st16(t_lane + T_P + c * 16, pp);
        tmem_st16(t_lane + T_DS + c * 16, ds);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(p_full);
    }
    if (ok && n_t > 0) {
      const bool got = mbar_wait(pv_done, (n_t - 1) & 1, abort_flag, p.err, kErrTimeoutEpilogue);
      ok = __all_sync(0xffffffffu, got);
    }
    if (ok) {
      tc_fence_after_sync();
      uint32_t a0[32], a1[32];
      const int64_t row = tile_row + r;
      if (KV) {
        // dV (no scale) and dK (times 1 / sqrt(hd)) of key row r
        uint32_t dv[64], dk[64];
        tmem_ld32(t_lane + T_ACC0, a0);
        tmem_ld32(t_lane + T_ACC0 + 32, a1);
        tmem_ld_wait(a0);
        tmem_ld_wait(a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          dv[i] = a0[i];
          dv[32 + i] = a1[i];
        }
        tmem_ld32(t_lane + T_ACC1, a0);
        tmem_ld32(t_lane + T_ACC1 + 32, a1);
        tmem_ld_wait(a0);
        tmem_ld_wait(a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          dk[i] = a0[i];
          dk[32 + i] = a1[i];
        }
        if (my_row < len) {
          store_row64(p.dqkv + row * 3 * D + col_k, dk, p.scale);
          store_row64(p.dqkv + row * 3 * D + col_v, dv, 1.0f);
        }
      } else {
        uint32_t dq[64];
        tmem_ld32(t_lane + T_ACC0, a0);
        tmem_ld32(t_lane + T_ACC0 + 32, a1);
        tmem_ld_wait(a0);
        tmem_ld_wait(a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          dq[i] = a0[i];
          dq[32 + i] = a1[i];
        }
        if (my_row < len) store_row64(p.dqkv + row * 3 * D + col_q, dq, p.scale);
      }
    }
    (void)et;
  }

  // Teardown: TMEM is released only after every warp has finished with it.
  tc_fence_before_sync();
  __syncwarp();
  if (lane == 0) mbar_arrive(teardown);
  {
    volatile int never = 0;
    mbar_wait(teardown, 0, &never, p.err, kErrTimeoutEpilogue);
  }
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}

// rowdot[h, p] = sum_j do[p, h*64 + j] * o[p, h*64 + j]: one warp per row, two lanes per head.
__global__ void k_attn_rowdot(const __nv_bfloat16* __restrict__ dout, const __nv_bfloat16* __restrict__ out,
                              float* __restrict__ rowdot, int64_t P, int H, int64_t ld) {
  grid_dependency_wait();
  launch_dependents();
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= P) return;
  const int D = H * HD;
  for (int h0 = 0; h0 < H; h0 += 16) {
    const int h = h0 + (lane >> 1);
    float acc = 0.0f;
    if (h < H) {
      const uint4* a = reinterpret_cast<const uint4*>(dout + row * D + h * HD + (lane & 1) * 32);
      const uint4* b = reinterpret_cast<const uint4*>(out + row * D + h * HD + (lane & 1) * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 x = a[q], y = b[q];
        acc += bf16_lo(x.x) * bf16_lo(y.x) + bf16_hi(x.x) * bf16_hi(y.x) + bf16_lo(x.y) * bf16_lo(y.y) +
               bf16_hi(x.y) * bf16_hi(y.y) + bf16_lo(x.z) * bf16_lo(y.z) + bf16_hi(x.z) * bf16_hi(y.z) +
               bf16_lo(x.w) * bf16_lo(y.w) + bf16_hi(x.w) * bf16_hi(y.w);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    if (h < H && (lane & 1) == 0) rowdot[static_cast<int64_t>(h) * ld + row] = acc;
  }
}

}  // namespace

cudaError_t launch_attention_bwd_tc(const CUtensorMap* tm_qkv, const CUtensorMap* tm_do, const AttnSchedule& kv_sched,
                                    const AttnSchedule& q_sched, const void* out, const void* dout, const float* lse,
                                    float* rowdot, int64_t lse_ld, void* dqkv, int64_t P, int H, int D, uint32_t* err,
                                    cudaStream_t s) {
  static unsigned long long attr_set_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(k_attn_bwd_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(k_attn_bwd_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set_mask |= 1ull << dev;
  }
  if (P == 0) return cudaSuccess;
  if (D != H * HD) return cudaErrorInvalidValue;
  const int64_t blocks = (P * 32 + 255) / 256;
  e = launch_pdl(k_attn_rowdot, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
                 static_cast<const __nv_bfloat16*>(dout), static_cast<const __nv_bfloat16*>(out), rowdot, P, H, lse_ld);
  if (e != cudaSuccess) return e;
  BwdParams p;
  p.n_heads = H;
  p.vision_dim = D;
  p.lse_ld = lse_ld;
  p.c_log2 = 1.4426950408889634f / 8.0f;  // log2(e) / sqrt(64)
  p.scale = 0.125f;
  p.lse = lse;
  p.rowdot = rowdot;
  p.dqkv = static_cast<__nv_bfloat16*>(dqkv);
  p.err = err;
  e = launch_pdl(k_attn_bwd_tc<true>, dim3(static_cast<unsigned>(kv_sched.n_items), static_cast<unsigned>(H)),
                 dim3(kThreads), SMEM_BYTES, s, *tm_qkv, *tm_do, kv_sched, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_attn_bwd_tc<false>, dim3(static_cast<unsigned>(q_sched.n_items), static_cast<unsigned>(H)),
                    dim3(kThreads), SMEM_BYTES, s, *tm_qkv, *tm_do, q_sched, p);
}

}  // namespace dsv4v
