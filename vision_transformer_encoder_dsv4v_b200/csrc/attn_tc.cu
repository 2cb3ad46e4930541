// Varlen full (bidirectional) attention on tcgen05, head_dim 64.
//
// One CTA per work item (image, one or two 128-query tiles A and B, head); items are scheduled
// longest image first.  Both query tiles of an item share every K/V tile that the producer
// loads.  For each 128-key tile j of the image and each query tile X of the item:
//   S_X = Q_X K_j^T            tcgen05.mma M=128 N=128 K=64, fp32 into TMEM
//   P_X = exp2(S_X c - m_X)    softmax warpgroup X, one query row per thread, written back to
//                             TMEM as bf16 (two keys per 32-bit column)
//   O_X += P_X V_j             tcgen05.mma M=128 N=64 K=128, A (= P) read from TMEM, V read
//                             MN-major from the natural [keys, hd] smem tile; O_X stays in TMEM
//                             for the whole key loop
// The row max m_X is raised lazily: only when a row's running max exceeds m_X by more than
// kRescaleLog2 (log2 units) are m_X, that row of O_X and its sum rescaled.  Otherwise the stale
// max is kept, which bounds P by 2^kRescaleLog2 and changes nothing but rounding.
// Keys past the end of the image are masked; query rows past it are computed but not stored.
//
// Warp roles: warp 0 TMA producer (Q once, K/V rings), warp 1 TMEM owner + MMA issuer of tile A,
// warp 2 MMA issuer of tile B, warp 3 idle, warps 4..7 softmax of tile A, warps 8..11 softmax of
// tile B.  Warp w reads TMEM lanes
// 32 (w % 4) .. +31, so every softmax thread owns one full query row of its tile (128 scores in
// registers).  The first warpgroup gives registers to the softmax warpgroups (setmaxnreg:
// 128 x 56 + 256 x 224 = 384 x 168, the launch's total).  The two softmax warpgroups share no
// barrier and drift apart, so that one's MUFU work overlaps the other's FMA work on each SM
// sub-partition.
//
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,320) O_B [320,384) P_A [384,448) P_B [448,512).
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

namespace {

constexpr int HD = 64;
constexpr int TQ = 128;                // queries per tile
constexpr int TK = 128;                // keys per tile
constexpr int KS = 4;                  // K ring depth
constexpr int VS = 4;                  // V ring depth
constexpr int TILE_BYTES = TK * HD * 2;  // 16 KB (Q, K or V tile)
constexpr int OFF_Q = 0;               // Q_A, Q_B
constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + VS * TILE_BYTES;
constexpr int OFF_XCHG = OFF_BAR + 512;  // split mode: each warpgroup's row max and sum (2 x 128 x 2 floats)
constexpr int SMEM_BYTES = 1024 + OFF_XCHG + 2048;
constexpr int kSoftmaxWarps = 8;
constexpr int kFirstSoftmaxWarp = 4;
constexpr int kRegsControl = 56;    // warpgroup 0 after setmaxnreg
constexpr int kRegsSoftmax = 224;   // softmax warpgroups after setmaxnreg
constexpr int kThreads = (kFirstSoftmaxWarp + kSoftmaxWarps) * 32;
constexpr int TMEM_COLS = 512;
constexpr uint32_t T_S = 0, T_O = 256, T_P = 384;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kPolyPerEight = 0;    // exponential pairs per eight computed on the FMA pipe (0: all on MUFU)

// Which exponential pairs (index i = column / 2) use the FMA-pipe polynomial.
__host__ __device__ constexpr bool poly_pair(int i) {
  return kPolyPerEight == 2   ? (i & 3) == 3
         : kPolyPerEight == 3 ? ((i & 7) == 2 || (i & 7) == 5 || (i & 7) == 7)
         : kPolyPerEight == 4 ? (i & 1) == 1
         : kPolyPerEight == 1 ? (i & 7) == 7
                              : false;
}

struct Params {
  int n_heads, vision_dim, pair;
  int split;  // one query tile per item: its key tiles alternate between the two warpgroups
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;       // optional [H, lse_ld]: log2 of each row's softmax denominator, in the units of
  int64_t lse_ld;   // s * scale_log2 (so that P = 2^(s scale_log2 - lse)); NULL: not written
  uint32_t* err;
};

// 2^x on the MUFU pipe (flushes results below 2^-126 to zero).
__device__ __forceinline__ float ex2_mufu(float x) { return ex2_approx(x); }

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for two x <= 0 at once on the FMA pipe, used for kPolyPerEight softmax exponential pairs
// in eight so that the MUFU pipe is not the only one doing them (none by default: with two
// softmax warpgroups per SM the MUFU pipe alone measured faster).  Range reduction x = n + f with
// n = round(x) (the 1.5 * 2^23 rounding trick) and f in [-1/2, 1/2]; 2^f by a cubic fitted here
// for minimum relative error on that interval (max 7.5e-5, far below the bf16 rounding of P);
// 2^n is added to the exponent field.  Inputs below -125 (masked keys included) return 0.
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

template <int R>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
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
  uint64_t* s_full = v_empty + VS;   // [tile]
  uint64_t* s_free = s_full + 2;     // [tile]
  uint64_t* p_full = s_free + 2;     // [tile]
  uint64_t* pv_done = p_full + 2;    // [tile]
  uint64_t* mma_done = pv_done + 2;  // [tile]
  uint64_t* teardown = mma_done + 2;  // one arrival per warp once its role is done
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(teardown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  int img, local;
  find_item(sched, blockIdx.x, img, local);
  const int row0 = sched.img_row0[img];
  const int len = sched.img_len[img];
  const int n_qt = (len + TQ - 1) / TQ;
  const int q_pair = local / p.n_heads;
  const int head = local - q_pair * p.n_heads;
  const int q_tile = q_pair * p.pair;
  const int n_tiles = min(p.pair, n_qt - q_tile);  // 1 or 2 query tiles in this item
  const int n_kv = (len + TK - 1) / TK;
  const int q_row = row0 + q_tile * TQ;
  // Split mode: one query tile; issuer/warpgroup x takes key tiles x, x + 2, x + 4, ... with its
  // own S, P and O in TMEM and its own running max and sum, and the two partial results are
  // combined at the end.  Otherwise group x owns query tile x and every key tile.
  const bool split = p.split != 0 && n_tiles == 1;
  const int n_groups = split ? 2 : n_tiles;
  const int kv_step = split ? 2 : 1;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], split ? 1 : n_tiles);  // released by every issuer that reads the slot
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], split ? 1 : n_tiles);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 128);
      mbar_init(&p_full[b], 128);
      mbar_init(&pv_done[b], 1);
    }
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    mbar_init(teardown, kThreads / 32);
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

  static_assert(kThreads == 384 && 128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * 168,
                "register split exceeds the launch's register total");
  if (warp < kFirstSoftmaxWarp) {
    regs_dec<kRegsControl>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      grid_dependency_wait();
      const int col_q = head * HD, col_k = p.vision_dim + head * HD, col_v = 2 * p.vision_dim + head * HD;
      mbar_arrive_expect_tx(q_full, n_tiles * TILE_BYTES);
      for (int x = 0; x < n_tiles; ++x)
        tma_load_2d(smem + OFF_Q + x * TILE_BYTES, &tm_qkv, q_full, col_q, q_row + x * TQ);
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
  } else if (warp - 1 < n_groups) {
    // ------------------------------------------------------------------ MMA issuers
    // Warp 1 issues the products of group A, warp 2 those of group B, so that neither waits for
    // the other's softmax; the K/V slots are released by one commit from each issuer that
    // reads them.
    if (lane == 0) {
      const int x = warp - 1;
      constexpr uint32_t idesc_s = idesc_bf16(TQ, TK, false);
      constexpr uint32_t idesc_pv = idesc_bf16(TQ, HD, true);  // V is MN-major (hd contiguous)
      const uint64_t qd = sdesc_sw128(smem_u32(smem + OFF_Q + (split ? 0 : x) * TILE_BYTES), 16, 1024);
      const uint32_t d_s = tmem_base + T_S + static_cast<uint32_t>(x * TK);
      const uint32_t d_o = tmem_base + T_O + static_cast<uint32_t>(x * HD);
      const uint32_t a_p = tmem_base + T_P + static_cast<uint32_t>(x * (TK / 2));
      auto issue_s = [&](int j) {
        const uint64_t kd = sdesc_sw128(smem_u32(smem + OFF_K + (j % KS) * TILE_BYTES), 16, 1024);
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) umma_bf16(d_s, qd + 2 * k, kd + 2 * k, idesc_s, k > 0 ? 1u : 0u);
        umma_commit(&s_full[x]);
        umma_commit(&k_empty[j % KS]);
      };
      // it: this group's iteration (its it-th key tile, global key tile j = x0 + it * kv_step).
      auto issue_pv = [&](int j, int it) {
        const uint32_t v_addr = smem_u32(smem + OFF_V + (j % VS) * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < TK / 16; ++kk) {
          // P: 16 keys = 8 TMEM columns; V: 16 keys = two 8-row groups of 1024 B.
          const uint64_t vd = sdesc_sw128(v_addr + kk * 2048, TILE_BYTES, 1024);
          umma_bf16_tmem_a(d_o, a_p + kk * 8, vd, idesc_pv, (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pv_done[x]);
        umma_commit(&v_empty[j % VS]);
      };
      const int x0 = split ? x : 0;
      bool ok = mbar_wait(q_full, 0, abort_flag, p.err, kErrTimeoutMma);
      if (ok && x0 < n_kv) {
        ok = mbar_wait(&k_full[x0 % KS], (x0 / KS) & 1, abort_flag, p.err, kErrTimeoutMma);
        if (ok) {
          tc_fence_after_sync();
          issue_s(x0);
        }
      }
      for (int j = x0, it = 0; j < n_kv && ok; j += kv_step, ++it) {
        if (j + kv_step < n_kv) {
          // S of the next key tile as soon as the softmax has this one's in registers.
          const int t = j + kv_step;
          ok = mbar_wait(&k_full[t % KS], (t / KS) & 1, abort_flag, p.err, kErrTimeoutMma) &&
               mbar_wait(&s_free[x], it & 1, abort_flag, p.err, kErrTimeoutMma);
          if (!ok) break;
          tc_fence_after_sync();
          issue_s(t);
        }
        ok = mbar_wait(&v_full[j % VS], (j / VS) & 1, abort_flag, p.err, kErrTimeoutMma) &&
             mbar_wait(&p_full[x], it & 1, abort_flag, p.err, kErrTimeoutMma);
        if (!ok) break;
        tc_fence_after_sync();
        issue_pv(j, it);
      }
      umma_commit(&mma_done[x]);
      volatile int never = 0;
      mbar_wait(&mma_done[x], 0, &never, p.err, kErrTimeoutMma);
    }
    __syncwarp();
  }
  } else if (regs_inc<kRegsSoftmax>(), (warp - kFirstSoftmaxWarp) / 4 < n_groups) {
    // ------------------------------------------------------------------ softmax + output
    const int x = (warp - kFirstSoftmaxWarp) >> 2;  // group of this warpgroup
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t t_s = t_lane + T_S + static_cast<uint32_t>(x * TK);
    const uint32_t t_o = t_lane + T_O + static_cast<uint32_t>(x * HD);
    const uint32_t t_p = t_lane + T_P + static_cast<uint32_t>(x * (TK / 2));
    float m_used = -INFINITY, l_run = 0.0f;
    bool ok = true;
    grid_dependency_wait();
    const int x0 = split ? x : 0;
    int n_it = 0;  // key tiles this group processed
    for (int kt = x0; kt < n_kv; kt += kv_step, ++n_it) {
      const int j = n_it;  // this group's iteration (barrier phases)
      bool got = mbar_wait(&s_full[x], j & 1, abort_flag, p.err, kErrTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      // Columns 0..63 first; 64..127 load while the first half's max is taken.
      uint32_t s[TK];
      tmem_ld_cols<2>(t_s, s);
      tmem_ld_issue<2>(t_s + 64, s + 64);
      const int valid = len - kt * TK;
      if (valid < TK / 2) {
#pragma unroll
        for (int c = 0; c < TK / 2; ++c)
          if (c >= valid) s[c] = 0xFF800000u;  // -inf
      }
      // Row max with eight independent chains of three-input max.
      float m8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) m8[u] = fmaxf(__uint_as_float(s[u]), __uint_as_float(s[8 + u]));
#pragma unroll
      for (int c = 16; c < TK / 2; c += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u) m8[u] = max3(m8[u], __uint_as_float(s[c + u]), __uint_as_float(s[c + 8 + u]));
      tmem_ld_wait_pin<2>(s + 64);
      tc_fence_before_sync();
      mbar_arrive(&s_free[x]);  // S is in registers: the next S may overwrite it
      if (valid < TK) {
#pragma unroll
        for (int c = TK / 2; c < TK; ++c)
          if (c >= valid) s[c] = 0xFF800000u;
      }
#pragma unroll
      for (int c = TK / 2; c < TK; c += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u) m8[u] = max3(m8[u], __uint_as_float(s[c + u]), __uint_as_float(s[c + 8 + u]));
      const float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
      const float m_cand = mx * p.scale_log2;
      const bool raise = m_cand > m_used + kRescaleLog2;
      const float m_new = raise ? m_cand : m_used;
      const float alpha = raise ? ex2_mufu(m_used - m_new) : 1.0f;  // 0 on the first tile
      m_used = m_new;
      // P = 2^(s c - m), some exponential pairs on the FMA pipe interleaved with the MUFU ones;
      // the bf16 pairs are packed in place into s[0 .. TK/2).  They are computed before waiting
      // for the previous P_X V product, which they overlap.
      // A ragged last key tile skips the 32-column chunks that hold no key (their P is zero).
      const uint64_t sc2 = pk2(p.scale_log2, p.scale_log2), nm2 = pk2(-m_new, -m_new);
      uint64_t l2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int ch = 0; ch < TK / 32; ++ch) {
        if (ch > 0 && 32 * ch >= valid) {
#pragma unroll
          for (int c = 32 * ch; c < 32 * ch + 32; c += 2) s[c >> 1] = 0u;
          continue;
        }
#pragma unroll
        for (int c = 32 * ch; c < 32 * ch + 32; c += 2) {
          float x0, x1, e0, e1;
          upk2(fma2(pk2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])), sc2, nm2), x0, x1);
          if (poly_pair(c >> 1)) {
            ex2_poly2(x0, x1, e0, e1);
          } else {
            e0 = ex2_mufu(x0);
            e1 = ex2_mufu(x1);
          }
          l2[(c >> 1) & 3] = add2(l2[(c >> 1) & 3], pk2(e0, e1));
          s[c >> 1] = pack_bf16x2(e0, e1);
        }
      }
      if (j > 0) {
        // P_X and O_X are free once the previous P_X V product has completed.
        got = mbar_wait(&pv_done[x], (j - 1) & 1, abort_flag, p.err, kErrTimeoutEpilogue);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
      }
      tmem_st32(t_p, s);
      tmem_st32(t_p + 32, s + 32);
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        uint32_t o[HD];
        tmem_ld_cols<HD / 32>(t_o, o);
        const uint64_t al2 = pk2(alpha, alpha);
#pragma unroll
        for (int c = 0; c < HD; c += 2) {
          float a0, a1;
          upk2(mul2(pk2(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), al2), a0, a1);
          o[c] = __float_as_uint(a0);
          o[c + 1] = __float_as_uint(a1);
        }
        tmem_st32(t_o, o);
        tmem_st32(t_o + 32, o + 32);
      }
      float la, lb, lc, ld, le, lf, lg, lh;
      upk2(l2[0], la, lb);
      upk2(l2[1], lc, ld);
      upk2(l2[2], le, lf);
      upk2(l2[3], lg, lh);
      l_run = l_run * alpha + (((la + lb) + (lc + ld)) + ((le + lf) + (lg + lh)));
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(&p_full[x]);
    }
    if (ok && n_it > 0) {
      const bool got = mbar_wait(&pv_done[x], (n_it - 1) & 1, abort_flag, p.err, kErrTimeoutEpilogue);
      ok = __all_sync(0xffffffffu, got);
    }
    float* xchg = reinterpret_cast<float*>(smem + OFF_XCHG);
    if (split) {
      // The two groups swap their row max and sum through shared memory and each writes half of
      // the output columns, [32 x, 32 x + 32), from both groups' O (same TMEM lane = same row):
      //   O = O_0 2^(m_0 - m) + O_1 2^(m_1 - m),  l = l_0 2^(m_0 - m) + l_1 2^(m_1 - m).
      const bool own = ok && n_it > 0;
      xchg[x * 256 + r] = own ? m_used : -INFINITY;
      xchg[x * 256 + 128 + r] = own ? l_run : 0.0f;
      tc_fence_before_sync();
      named_barrier_sync(3, 256);
      tc_fence_after_sync();
      const float m_b = xchg[(1 - x) * 256 + r], l_b = xchg[(1 - x) * 256 + 128 + r];
      constexpr int HH = HD / 2;
      const uint32_t col = static_cast<uint32_t>(x * HH);
      uint32_t oa[HH], ob[HH];
      if (own) tmem_ld_cols<HH / 32>(t_o + col, oa);
      if (__any_sync(0xffffffffu, l_b > 0.0f))
        tmem_ld_cols<HH / 32>(t_lane + T_O + static_cast<uint32_t>((1 - x) * HD) + col, ob);
      const float m = fmaxf(own ? m_used : -INFINITY, m_b);
      const float fa = own ? ex2_mufu(m_used - m) : 0.0f;
      const float fb = l_b > 0.0f ? ex2_mufu(m_b - m) : 0.0f;
      const float l_tot = (own ? l_run * fa : 0.0f) + l_b * fb;
      const int qi = q_tile * TQ + r;
      if (qi < len && l_tot > 0.0f) {
        if (x == 0 && p.lse) p.lse[static_cast<int64_t>(head) * p.lse_ld + row0 + qi] = m + __log2f(l_tot);
        const float inv_l = 1.0f / l_tot;
        const float ga = fa * inv_l, gb = fb * inv_l;
        float o[HH];
#pragma unroll
        for (int c = 0; c < HH; ++c) {
          const float va = own ? __uint_as_float(oa[c]) * ga : 0.0f;
          o[c] = l_b > 0.0f ? fmaf(__uint_as_float(ob[c]), gb, va) : va;
        }
        uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(row0 + qi) * p.vision_dim + head * HD + col);
#pragma unroll
        for (int q = 0; q < HH / 8; ++q) {
          uint4 v;
          v.x = pack_bf16x2(o[8 * q + 0], o[8 * q + 1]);
          v.y = pack_bf16x2(o[8 * q + 2], o[8 * q + 3]);
          v.z = pack_bf16x2(o[8 * q + 4], o[8 * q + 5]);
          v.w = pack_bf16x2(o[8 * q + 6], o[8 * q + 7]);
          dst[q] = v;
        }
      }
    } else if (ok) {
      tc_fence_after_sync();
      uint32_t o[HD];
      tmem_ld_cols<HD / 32>(t_o, o);
      const int qi = (q_tile + x) * TQ + r;
      if (qi < len && p.lse) p.lse[static_cast<int64_t>(head) * p.lse_ld + row0 + qi] = m_used + __log2f(l_run);
      if (qi < len) {
        const float inv_l = 1.0f / l_run;
        uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(row0 + qi) * p.vision_dim + head * HD);
#pragma unroll
        for (int q = 0; q < HD / 8; ++q) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
          dst[q] = v;
        }
      }
    }
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
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attention_tc(const CUtensorMap* tm_qkv, const AttnSchedule& sched, int n_heads, int vision_dim,
                                void* out, uint32_t* err, cudaStream_t s, float* lse, int64_t lse_ld) {
  static unsigned long long attr_set_mask = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(attr_set_mask & (1ull << dev))) {
    // setmaxnreg.inc waits until the block has the registers it asks for: refuse to launch if
    // the build gave the kernel fewer registers per thread than the split assumes.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k_attn_tc);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * kThreads < 128 * kRegsControl + 256 * kRegsSoftmax) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev < 64) attr_set_mask |= 1ull << dev;
  }
  if (sched.n_items <= 0) return cudaSuccess;
  if (sched.pair != 1 && sched.pair != 2) return cudaErrorInvalidValue;
  Params p;
  p.n_heads = n_heads;
  p.vision_dim = vision_dim;
  p.pair = sched.pair;
  p.split = sched.split;
  p.scale_log2 = 1.4426950408889634f / 8.0f;  // log2(e) / sqrt(64)
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.lse_ld = lse_ld;
  p.err = err;
  return launch_pdl(k_attn_tc, dim3(sched.n_items), dim3(kThreads), SMEM_BYTES, s, *tm_qkv, sched, p);
}

}  // namespace dsv4v
