// Varlen full (bidirectional) attention on tcgen05, head_dim 64.
//
// One CTA per work item (image, 128-query tile, head); items are scheduled longest image
// first.  For each 128-key tile j of the image:
//   S_j = Q K_j^T          tcgen05.mma M=128 N=128 K=64, fp32 into TMEM (two S buffers)
//   P_j = exp2(S_j * log2(e)/sqrt(hd) - m_j)   softmax warps, one query row per thread, written
//                          to smem as bf16 in the 128-byte-swizzled K-major layout
//   PV_j = P_j V_j         tcgen05.mma M=128 N=64 K=128 (V read MN-major straight from the
//                          natural [keys, hd] tile), fp32 into TMEM (two PV buffers)
//   O = O * exp2(m_{j-1} - m_j) + PV_j     in registers, one tile behind, so the tensor core
//                          computes S_{j+1} and PV_j while the softmax warps work on S_j.
// Keys past the end of the image are masked; query rows past it are computed but not stored.
//
// Warp roles: warp 0 TMA producer (Q once, K/V rings), warp 1 TMEM owner + MMA issuer,
// warps 2..9 softmax / output.  Warps w and w + 4 share the query rows of TMEM lane quadrant
// w % 4: the first takes keys 0..63 of each S tile and output columns 0..31, the second keys
// 64..127 and columns 32..63; they exchange row maxima (and at the end row sums) through shared
// memory at a pair barrier.
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

constexpr int HD = 64;
constexpr int TQ = 128;                // queries per CTA
constexpr int TK = 128;                // keys per tile
constexpr int KS = 3;                  // K ring depth
constexpr int VS = 3;                  // V ring depth
constexpr int TILE_BYTES = TK * HD * 2;  // 16 KB (Q, K or V tile)
constexpr int P_BYTES = TQ * TK * 2;     // 32 KB
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
constexpr int OFF_P = OFF_V + VS * TILE_BYTES;
constexpr int OFF_XCH = OFF_P + 2 * P_BYTES;  // [2 tiles][2 halves][128 rows] fp32 exchange
constexpr int OFF_BAR = OFF_XCH + 2 * 2 * 128 * 4;
constexpr int SMEM_BYTES = 1024 + OFF_BAR + 512;
constexpr int kSoftmaxWarps = 8;  // two per query row: one per 64-key half of each S tile
constexpr int kThreads = 64 + kSoftmaxWarps * 32;
constexpr int TMEM_COLS = 512;  // S0 [0,128) S1 [128,256) PV0 [256,320) PV1 [320,384)

struct Params {
  int n_heads, vision_dim;
  float scale_log2;
  __nv_bfloat16* out;
  uint32_t* err;
};

// 2^x on the MUFU pipe (flushes results below 2^-126 to zero).
__device__ __forceinline__ float ex2_mufu(float x) { return ex2_approx(x); }

// 2^x for x <= 0 on the FMA pipe, used for a quarter of the softmax exponentials so that the
// MUFU pipe is not the only one doing them.  Range reduction x = n + f with n = round(x) (the
// 1.5 * 2^23 rounding trick) and f in [-1/2, 1/2]; 2^f by a cubic fitted here for minimum
// relative error on that interval (max 7.5e-5, far below the bf16 rounding of P); 2^n is added
// to the exponent field.  Inputs below -125 (masked keys included) return 0.
__device__ __forceinline__ float ex2_poly(float x) {
  const float xc = fmaxf(x, -125.0f);
  const float t = xc + 12582912.0f;
  const float n = t - 12582912.0f;
  const float f = xc - n;
  const float p = fmaf(fmaf(fmaf(0.0551716573536396f, f, 0.2426111400127411f), f, 0.6932609677314758f), f,
                       0.9999280571937561f);
  const int ni = __float_as_int(t) - 0x4B400000;
  const float r = __int_as_float(__float_as_int(p) + static_cast<int>(static_cast<unsigned>(ni) << 23));
  return x < -125.0f ? 0.0f : r;
}

// Packed pairs of fp32 (one 64-bit register pair) for the sm_100 f32x2 arithmetic.
__device__ __forceinline__ uint64_t pk2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ex2_poly on two elements at once with packed arithmetic (same reduction and cubic).
__device__ __forceinline__ void ex2_poly2(float x0, float x1, float& y0, float& y1) {
  const uint64_t xc = pk2(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t magic = pk2(12582912.0f, 12582912.0f);
  const uint64_t t = add2(xc, magic);
  const uint64_t f = sub2(xc, sub2(t, magic));
  uint64_t q = fma2(pk2(0.0551716573536396f, 0.0551716573536396f), f, pk2(0.2426111400127411f, 0.2426111400127411f));
  q = fma2(q, f, pk2(0.6932609677314758f, 0.6932609677314758f));
  q = fma2(q, f, pk2(0.9999280571937561f, 0.9999280571937561f));
  float t0, t1, q0, q1;
  upk2(t, t0, t1);
  upk2(q, q0, q1);
  const unsigned n0 = static_cast<unsigned>(__float_as_int(t0) - 0x4B400000);
  const unsigned n1 = static_cast<unsigned>(__float_as_int(t1) - 0x4B400000);
  y0 = x0 < -125.0f ? 0.0f : __int_as_float(__float_as_int(q0) + static_cast<int>(n0 << 23));
  y1 = x1 < -125.0f ? 0.0f : __int_as_float(__float_as_int(q1) + static_cast<int>(n1 << 23));
}

__device__ __forceinline__ void find_item(const AttnSchedule& s, int item, int& img, int& local) {
  int lo = 0, hi = s.n_images - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s.item_start[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  img = lo;
  local = item - s.item_start[lo];
}

__global__ void __launch_bounds__(kThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ AttnSchedule sched,
              const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + KS;
  uint64_t* v_full = k_empty + KS;
  uint64_t* v_empty = v_full + VS;
  uint64_t* s_full = v_empty + VS;   // [2]
  uint64_t* p_full = s_full + 2;     // [2]
  uint64_t* pv_full = p_full + 2;    // [2]
  uint64_t* pv_empty = pv_full + 2;  // [2]
  uint64_t* mma_done = pv_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int img, local;
  find_item(sched, blockIdx.x, img, local);
  const int row0 = sched.img_row0[img];
  const int len = sched.img_len[img];
  const int q_tile = local / p.n_heads;
  const int head = local - q_tile * p.n_heads;
  const int n_kv = (len + TK - 1) / TK;
  const int q_row = row0 + q_tile * TQ;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], kSoftmaxWarps * 32);
      mbar_init(&pv_full[b], 1);
      mbar_init(&pv_empty[b], kSoftmaxWarps * 32);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm_qkv);
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
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
      const int col_q = head * HD, col_k = p.vision_dim + head * HD, col_v = 2 * p.vision_dim + head * HD;
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      tma_load_2d(smem + OFF_Q, &tm_qkv, q_full, col_q, q_row);
      int issued_k = 0, issued_v = 0;
      for (int t = 0; t < n_kv; ++t) {
        if (!mbar_wait(&k_empty[t % KS], ((t / KS) & 1) ^ 1, abort_flag, p.err, kErrTimeoutProducer)) break;
        mbar_arrive_expect_tx(&k_full[t % KS], TILE_BYTES);
        tma_load_2d(smem + OFF_K + (t % KS) * TILE_BYTES, &tm_qkv, &k_full[t % KS], col_k, row0 + t * TK);
        issued_k = t + 1;
        if (!mbar_wait(&v_empty[t % VS], ((t / VS) & 1) ^ 1, abort_flag, p.err, kErrTimeoutProducer)) break;
        mbar_arrive_expect_tx(&v_full[t % VS], TILE_BYTES);
        tma_load_2d(smem + OFF_V + (t % VS) * TILE_BYTES, &tm_qkv, &v_full[t % VS], col_v, row0 + t * TK);
        issued_v = t + 1;
      }
      // Let copies still in flight land before exit (returns at once in the normal path).
      volatile int never = 0;
      mbar_wait(q_full, 0, &never, p.err, kErrTimeoutProducer);
      for (int t = (issued_k > KS ? issued_k - KS : 0); t < issued_k; ++t)
        mbar_wait(&k_full[t % KS], (t / KS) & 1, &never, p.err, kErrTimeoutProducer);
      for (int t = (issued_v > VS ? issued_v - VS : 0); t < issued_v; ++t)
        mbar_wait(&v_full[t % VS], (t / VS) & 1, &never, p.err, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(TQ, TK, false);
      constexpr uint32_t idesc_pv = idesc_bf16(TQ, HD, true);  // V is MN-major (hd contiguous)
      const uint32_t q_addr = smem_u32(smem + OFF_Q);
      const uint32_t p_addr = smem_u32(smem + OFF_P);
      bool ok = mbar_wait(q_full, 0, abort_flag, p.err, kErrTimeoutMma);
      tc_fence_after_sync();
      auto issue_s = [&](int j) -> bool {
        if (!mbar_wait(&k_full[j % KS], (j / KS) & 1, abort_flag, p.err, kErrTimeoutMma)) return false;
        tc_fence_after_sync();
        const uint32_t k_addr = smem_u32(smem + OFF_K + (j % KS) * TILE_BYTES);
        const uint64_t qd = sdesc_sw128(q_addr, 16, 1024);
        const uint64_t kd = sdesc_sw128(k_addr, 16, 1024);
        const uint32_t d = tmem_base + static_cast<uint32_t>((j & 1) * TK);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) umma_bf16(d, qd + 2 * k, kd + 2 * k, idesc_s, k > 0 ? 1u : 0u);
        umma_commit(&k_empty[j % KS]);
        umma_commit(&s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && n_kv > 1) ok = issue_s(1);
      for (int j = 0; j < n_kv && ok; ++j) {
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1, abort_flag, p.err, kErrTimeoutMma)) break;
        if (j >= 2 && !mbar_wait(&pv_empty[j & 1], ((j - 2) >> 1) & 1, abort_flag, p.err, kErrTimeoutMma)) break;
        if (!mbar_wait(&v_full[j % VS], (j / VS) & 1, abort_flag, p.err, kErrTimeoutMma)) break;
        tc_fence_after_sync();
        const uint32_t v_addr = smem_u32(smem + OFF_V + (j % VS) * TILE_BYTES);
        const uint32_t pj = p_addr + (j & 1) * P_BYTES;
        const uint32_t d = tmem_base + 256u + static_cast<uint32_t>((j & 1) * HD);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          // P: two 64-key swizzle atoms of 16 KB; V: 16 keys = two 8-row groups of 1024 B.
          const uint64_t pd = sdesc_sw128(pj + (kk >> 2) * (TQ * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t vd = sdesc_sw128(v_addr + kk * 2048, TILE_BYTES, 1024);
          umma_bf16(d, pd, vd, idesc_pv, kk > 0 ? 1u : 0u);
        }
        umma_commit(&v_empty[j % VS]);
        umma_commit(&pv_full[j & 1]);
        if (j + 2 < n_kv) ok = issue_s(j + 2);
      }
      umma_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never, p.err, kErrTimeoutMma);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + output
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quad * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t pair_bar = 2 + quad;  // named barrier of warps (quad + 2 or quad + 6) and partner
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    uint8_t* p_smem = smem + OFF_P;
    float* xch = reinterpret_cast<float*>(smem + OFF_XCH);
    float o[HD / 2];
#pragma unroll
    for (int c = 0; c < HD / 2; ++c) o[c] = 0.0f;
    float m_run = -INFINITY, l_run = 0.0f, alpha_prev = 0.0f;
    bool ok = true;
    grid_dependency_wait();
    auto accumulate_pv = [&](int j, float alpha) -> bool {
      bool got = mbar_wait(&pv_full[j & 1], (j >> 1) & 1, abort_flag, p.err, kErrTimeoutEpilogue);
      got = __all_sync(0xffffffffu, got);
      if (!got) return false;
      tc_fence_after_sync();
      uint32_t a[32];
      tmem_ld32(t_lane + 256u + static_cast<uint32_t>((j & 1) * HD + half * 32), a);
      tmem_ld_wait(a);
      const uint64_t al2 = pk2(alpha, alpha);
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const uint64_t r2 = fma2(pk2(o[c], o[c + 1]), al2, pk2(__uint_as_float(a[c]), __uint_as_float(a[c + 1])));
        upk2(r2, o[c], o[c + 1]);
      }
      tc_fence_before_sync();
      mbar_arrive(&pv_empty[j & 1]);
      return true;
    };
    for (int j = 0; j < n_kv; ++j) {
      bool got = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag, p.err, kErrTimeoutEpilogue);
      got = __all_sync(0xffffffffu, got);
      uint32_t s[TK / 2];
      float mx = -INFINITY;
      if (got) {
        tc_fence_after_sync();
        const uint32_t ts = t_lane + static_cast<uint32_t>((j & 1) * TK + half * (TK / 2));
        tmem_ld32(ts + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld32(ts + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld_wait(*reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        const int valid = min(TK, len - j * TK) - half * (TK / 2);  // keys of this half inside the image
        if (valid < TK / 2) {
#pragma unroll
          for (int c = 0; c < TK / 2; ++c)
            if (c >= valid) s[c] = 0xFF800000u;  // -inf
        }
        // Row max over this half with eight independent chains.
        float m8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) m8[u] = __uint_as_float(s[u]);
#pragma unroll
        for (int c = 8; c < TK / 2; c += 8)
#pragma unroll
          for (int u = 0; u < 8; ++u) m8[u] = fmaxf(m8[u], __uint_as_float(s[c + u]));
        mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
      }
      float* xm = xch + (j & 1) * 256;  // double-buffered by tile parity
      xm[half * 128 + r] = mx;
      if (!named_barrier_and(pair_bar, 64, got)) {
        ok = false;
        break;
      }
      mx = fmaxf(mx, xm[(1 - half) * 128 + r]);
      const float m_new = fmaxf(m_run, mx * p.scale_log2);
      const float alpha = ex2_mufu(m_run - m_new);
      const float neg_m = -m_new;
      // This half's 64 keys are swizzle atom `half` of the P row.  One exponential pair in four
      // runs on the FMA pipe, interleaved with the MUFU ones so that both pipes stay busy; the
      // scale-subtract, the row sum and the cubic use packed f32x2 arithmetic.
      uint8_t* prow = p_smem + (j & 1) * P_BYTES + half * (TQ * 128) + r * 128;
      const uint64_t sc2 = pk2(p.scale_log2, p.scale_log2), nm2 = pk2(neg_m, neg_m);
      uint64_t l2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int c16 = 0; c16 < TK / 16; ++c16) {
        float e[8];
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          float x0, x1;
          upk2(fma2(pk2(__uint_as_float(s[c16 * 8 + u]), __uint_as_float(s[c16 * 8 + u + 1])), sc2, nm2), x0, x1);
          if (u == 6) {
            ex2_poly2(x0, x1, e[u], e[u + 1]);
          } else {
            e[u] = ex2_mufu(x0);
            e[u + 1] = ex2_mufu(x1);
          }
          l2[u >> 1] = add2(l2[u >> 1], pk2(e[u], e[u + 1]));
        }
        uint4 pk;
        pk.x = pack_bf16x2(e[0], e[1]);
        pk.y = pack_bf16x2(e[2], e[3]);
        pk.z = pack_bf16x2(e[4], e[5]);
        pk.w = pack_bf16x2(e[6], e[7]);
        *reinterpret_cast<uint4*>(prow + ((c16 ^ (r & 7)) << 4)) = pk;
      }
      float la, lb, lc, ld, le, lf, lg, lh;
      upk2(l2[0], la, lb);
      upk2(l2[1], lc, ld);
      upk2(l2[2], le, lf);
      upk2(l2[3], lg, lh);
      const float sum = ((la + lb) + (lc + ld)) + ((le + lf) + (lg + lh));
      l_run = l_run * alpha + sum;
      m_run = m_new;
      fence_proxy_async_smem();  // generic-proxy P stores -> visible to the tensor core
      tc_fence_before_sync();
      mbar_arrive(&p_full[j & 1]);
      if (j >= 1 && !accumulate_pv(j - 1, alpha_prev)) {
        ok = false;
        break;
      }
      alpha_prev = alpha;
    }
    if (ok && n_kv > 0) ok = accumulate_pv(n_kv - 1, alpha_prev);
    // Row sum = sum of the two halves' sums (both are relative to the same running max).
    float* xl = xch + 512 - 256;  // reuse the exchange of tile parity 1 (its readers have passed)
    named_barrier_sync(pair_bar, 64);
    xl[half * 128 + r] = l_run;
    named_barrier_sync(pair_bar, 64);
    const float l_total = l_run + xl[(1 - half) * 128 + r];
    const int qi = q_tile * TQ + r;
    if (ok && qi < len) {
      const float inv_l = 1.0f / l_total;
      uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(row0 + qi) * p.vision_dim + head * HD + half * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16x2(o[8 * q + 0] * inv_l, o[8 * q + 1] * inv_l);
        v.y = pack_bf16x2(o[8 * q + 2] * inv_l, o[8 * q + 3] * inv_l);
        v.z = pack_bf16x2(o[8 * q + 4] * inv_l, o[8 * q + 5] * inv_l);
        v.w = pack_bf16x2(o[8 * q + 6] * inv_l, o[8 * q + 7] * inv_l);
        dst[q] = v;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attention_tc(const CUtensorMap* tm_qkv, const AttnSchedule& sched, int n_heads, int vision_dim,
                                void* out, uint32_t* err, cudaStream_t s) {
  static unsigned long long attr_set_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set_mask & (1ull << dev))) {
    e = cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set_mask |= 1ull << dev;
  }
  if (sched.n_items <= 0) return cudaSuccess;
  Params p;
  p.n_heads = n_heads;
  p.vision_dim = vision_dim;
  p.scale_log2 = 1.4426950408889634f / 8.0f;  // log2(e) / sqrt(64)
  p.out = static_cast<__nv_bfloat16*>(out);
  p.err = err;
  return launch_pdl(k_attn_tc, dim3(sched.n_items), dim3(kThreads), SMEM_BYTES, s, *tm_qkv, sched, p);
}

}  // namespace dsv4v
