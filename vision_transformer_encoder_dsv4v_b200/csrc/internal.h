// Host-side interface between the C ABI (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsv4v {

// ---------------------------------------------------------------------------- tcgen05 GEMM
// C[M, n_out] = A[M, K] . B[n, K]^T with a fused epilogue; bf16 operands, fp32 accumulation.
enum Epi : int {
  EPI_STORE = 0,     // out = acc
  EPI_RESID = 1,     // out = resid + acc          (out may alias resid)
  EPI_QKV_ROPE = 2,  // out = acc, columns < rot_cols rotated pairwise (j, j + 32) per 64-wide head
  EPI_SWIGLU = 3,    // out = silu(acc_gate) * acc_up; B = gate rows, B2 = up rows
  EPI_GELU = 4,      // out = gelu(acc + bias), gelu(z) = z (1 + erf(z / sqrt 2)) / 2
};

struct GemmPlan {
  int bn;        // MMA N per tile (SWIGLU: gate + up halves)
  int pair;      // 1: 256-row tiles on CTA pairs (tcgen05 cta_group::2), grid even; 0: 128-row tiles
  int ks;        // > 1 (residual, store, GELU epilogues): each tile is split along K over a cluster of ks
                 // CTAs, reduced through distributed shared memory (bn = 256; each CTA finishes
                 // 256 / ks columns)
  int splits;    // K splits per tile (fix-up by the last finisher)
  int tiles_m, tiles_n, kb_total, work, grid;
  size_t partial_bytes;  // fp32 scratch for split tiles
  int counters;          // tile counters needed (split tiles only)
};

// Row partial sums of x^2 a residual GEMM with this plan writes per row (one per column slice).
inline int norm_parts_of(const GemmPlan& p) { return p.tiles_n * (p.ks > 1 ? p.ks : 1); }

// Chooses tile width, CTA pairing and split count for a GEMM of this shape on `num_sms` SMs;
// plans whose split-tile partials exceed max_partial_bytes are not considered.
GemmPlan plan_gemm(int epi, int M, int n_out, int K, int num_sms, size_t max_partial_bytes = SIZE_MAX);
// Whole-tile plans (the grid divides the tile count) with 64-, 128- or 256-column tiles and no
// cluster split-K: what GemmArgs::mn_major supports.
GemmPlan plan_gemm_whole(int M, int n_out, int K, int num_sms);

struct GemmArgs {
  const CUtensorMap* tm_out;  // output [M, n_out] bf16, box 64 x 32 (TMA stores of the epilogue)
  const CUtensorMap* tm_xw;   // RESID with the next norm prepared: xw_out [M, n_out], box 64 x 32
  const CUtensorMap* tm_a;    // A [M, K], box 64 x 128
  const CUtensorMap* tm_b;    // B [n, K] (SWIGLU: w_gate), box 64 x bn (SWIGLU or pair: bn / 2)
  const CUtensorMap* tm_b2;   // SWIGLU: w_up, box 64 x bn / 2
  int M, K, n_out;
  void* out;
  int ldo;
  const void* resid;
  const float* cos;
  const float* sin;
  int rot_cols;
  float* partials;
  int* counters;
  uint32_t* err;
  // RMSNorm folded into the GEMM (norm(x) W^T = r_p ((x * w) W^T), r_p = 1/sqrt(mean x_p^2 + eps)):
  //  consumer side (QKV_ROPE, SWIGLU): A holds bf16(x * w); the epilogue scales row p by r_p,
  //   computed from norm_ss[p * norm_stride + i], i < norm_parts (partial sums of x_p^2);
  //   norm_ss == NULL: no scaling.
  //  producer side (RESID): besides x, the epilogue writes xw_out = bf16(x * xw_w) and the
  //   partial sums of x^2 of its columns to ss_out[p * ss_parts + n_tile]; xw_out == NULL: off.
  const float* norm_ss;
  int norm_parts, norm_stride;
  float norm_inv_d, norm_eps;
  void* xw_out;
  const float* xw_w;
  float* ss_out;
  int ss_parts;
  const float* bias;  // STORE: per-column fp32 bias added before rounding (NULL: none)
  // B (and B2) are weights that no kernel still in flight on the stream writes: their first
  // stages may be loaded before the dependency wait.  Otherwise (B produced by an earlier kernel
  // of the same call, as in the backward's weight gradients) every load waits.
  bool b_early;
  // Up to two ranges (the next GEMM's weights) that the CTAs prefetch into L2, a share each,
  // once their own operand loads are issued (NULL: none; 16-byte aligned, bytes a multiple of 16).
  const void* l2_next[2];
  size_t l2_next_bytes[2];
  // Operand major-ness (STORE epilogue; whole-tile plans, or cluster split-K when A is K-major): bit 0,
  // B is MN-major: tm_b describes the stored [K, n] matrix (n contiguous), box 64 x 64; bit 1, A
  // is MN-major: tm_a describes the stored [K, M] matrix, box 64 x 64; bit 2 (with bit 0), the
  // K extent of B continues in tm_b2 from K block kb_split on (B = [B1; B2] stacked along K).
  int mn_major;
  int kb_split;
};

cudaError_t launch_gemm_tc(int epi, const GemmPlan& plan, const GemmArgs& a, cudaStream_t s);

// ---------------------------------------------------------------------------- chain kernel
// Several dependent GEMM stages of the block in one persistent launch (chain.cu).  Stage tiles
// are 128 rows x bn columns, K in 64-element blocks, optionally split along K; a stage waits per
// 128-row tile for an earlier stage of the same launch (dep_stage), or for the kernels before
// the launch (dep_stage < 0).
constexpr int kChainMaxStages = 4;
constexpr int kChainMaxMaps = 20;
enum ChainEpi : int {
  CHAIN_RESID = 0,      // out = resid + acc; optionally xw = bf16(out * xw_w) and row sums of out^2
  CHAIN_SWIGLU = 1,     // out = silu(r acc_gate) * (r acc_up); B = gate rows, B2 = up rows (bn / 2 each)
  CHAIN_QKV_HEADS = 2,  // bn = 192: the q, k, v rows of head n; rows scaled by r, q and k rotated
};
struct ChainStage {
  int epi, bn, kb_total, tiles_m, tiles_n, splits, task_base;
  int dep_stage, dep_target;                   // counters of an earlier stage of the launch (-1: none)
  int map_a, map_b, map_b2, map_out, map_xw;   // indices into ChainParams::maps (-1: unused)
  int M, D;                                    // rows; vision_dim (head-blocked q|k|v output columns)
  const void* resid;                           // CHAIN_RESID: bf16 residual rows, row stride ldr
  int ldr;
  const float* cos;                            // CHAIN_QKV_HEADS: rotation tables [M, 32]
  const float* sin;
  const float* norm_ss;                        // folded norm, consumer side (NULL: r = 1)
  int norm_parts, norm_stride;
  const float* xw_w;                           // folded norm, producer side (map_xw >= 0)
  float* ss_out;
  int ss_parts;
  float* partials;                             // splits > 1: [tiles][splits - 1][128 * bn] fp32
  int* arrivals;                               // splits > 1: [tiles], zero between launches
  int* done;                                   // [tiles_m]: finished tiles per row tile, zero before the launch
};
struct ChainParams {
  CUtensorMap maps[kChainMaxMaps];
  ChainStage st[kChainMaxStages];
  int n_stages, n_maps, total_tasks;
  int ring_slots, slot_bytes;  // operand ring: slots of slot_bytes (>= every stage's A + B bytes,
                               // a multiple of 1024), ring_slots * slot_bytes <= chain_ring_bytes()
  float norm_inv_d, norm_eps;
  int* ticket;  // zero before the launch
  uint32_t* err;
};
cudaError_t launch_chain(const ChainParams& p, int grid, cudaStream_t s);
// Shared-memory bytes of the chain kernel's operand ring.
int chain_ring_bytes();

// ---------------------------------------------------------------------------- attention
constexpr int kMaxImages = 1024;

// Images in the order they are scheduled (longest first); item_start is the prefix sum of
// (query tiles x heads) in that order.
// Work items of the attention kernel: for each image (longest first) and head, its query tiles
// in groups of `pair` (1 or 2) 128-row tiles that share the K/V stream.
struct AttnSchedule {
  int n_images;
  int n_items;
  int pair;
  int split;  // pair == 1 only: the two softmax warpgroups of a CTA share its query tile's key tiles
  int item_start[kMaxImages + 1];
  int img_row0[kMaxImages];
  int img_len[kMaxImages];
};

// lse (optional, [n_heads, lse_ld] fp32): per row and head, log2 of the softmax denominator in
// the units of the scaled scores, P = 2^(q.k log2(e) / sqrt(hd) - lse).
cudaError_t launch_attention_tc(const CUtensorMap* tm_qkv, const AttnSchedule& sched, int n_heads, int vision_dim,
                                void* out, uint32_t* err, cudaStream_t s, float* lse = nullptr, int64_t lse_ld = 0);

// Attention backward on tcgen05 (attn_bwd_tc.cu): rowdot[h, p] = rowsum(dout * out) per head,
// then dK/dV (one CTA per key tile and head, kv_sched) and dQ (one CTA per query tile and head,
// q_sched) into dqkv [P, 3D].  lse / rowdot: [H, lse_ld] fp32, lse from launch_attention_tc.
cudaError_t launch_attention_bwd_tc(const CUtensorMap* tm_qkv, const CUtensorMap* tm_do, const AttnSchedule& kv_sched,
                                    const AttnSchedule& q_sched, const void* out, const void* dout, const float* lse,
                                    float* rowdot, int64_t lse_ld, void* dqkv, int64_t P, int H, int D, uint32_t* err,
                                    cudaStream_t s);

// ---------------------------------------------------------------------------- small kernels
// The first kernel of an entry point also clears the GEMM tile counters of the call
// (zero_ptr / zero_n; NULL / 0 when it has none to clear).
cudaError_t launch_rope_table(const int32_t* cu_dev, const int32_t* grid_dev, int n_images, int64_t P, int half,
                              float theta, float* cos_out, float* sin_out, cudaStream_t s, int* zero_ptr = nullptr,
                              int zero_n = 0);
cudaError_t launch_rmsnorm(bool bf16, const void* x, const float* w, void* y, int64_t rows, int d, float eps,
                           cudaStream_t s, int* zero_ptr = nullptr, int zero_n = 0);
cudaError_t launch_aligner_index(const int32_t* cu_dev, const int32_t* grid_dev, int n_images, int r,
                                 int64_t n_tokens, int32_t* src_out, cudaStream_t s, int* zero_ptr = nullptr,
                                 int zero_n = 0);
cudaError_t launch_zero_counters(int* ptr, int n, cudaStream_t s);
// Merged r x r window rows of bf16 patch rows: merged[t, s * d : (s + 1) * d] = x[src[t * r2 + s]],
// zeros where src < 0 (d a multiple of 8).
cudaError_t launch_merge_rows_bf16(const void* x, const int32_t* src, void* merged, int64_t n_tokens, int r2, int d,
                                   cudaStream_t s);
// LayerNorm of each patch row (weight and bias, fp32 math) written into its slot of the merged
// r x r window rows: merged[t, s * d : (s + 1) * d] = LN(x[src[t * r2 + s]]), zeros where
// src < 0.  bf16 or fp32 activations.
cudaError_t launch_ln_merge(bool bf16, const void* x, const int32_t* src, const float* w, const float* b, float eps,
                            void* merged, int64_t n_tokens, int r2, int d, cudaStream_t s);
cudaError_t launch_selftest_wait(uint64_t limit_ns, uint32_t* err, cudaStream_t s);
// Backward of the block (backward.cu).  All bf16 except the fp32 norm weights, their gradients,
// the rotation tables and the attention row statistics.
cudaError_t launch_rmsnorm_bwd(const void* x, const float* w, const void* dy, const void* d_in, void* dx,
                               float* partial, int parts, float* dw, int64_t rows, int d, float eps, cudaStream_t s);
cudaError_t launch_swiglu_bwd(const void* g, const void* u, const void* dh, void* dgu, void* h, int64_t rows, int f,
                              int sms, cudaStream_t s);
cudaError_t launch_rotary_bwd(void* dqkv, const float* cos, const float* sin, int64_t P, int D, int hd, int sms,
                              cudaStream_t s);
// Image-token bridge (bridge.cu).  Positions per CTA of the merge and the visibility scan;
// counts holds one int4 per chunk of that many positions.
constexpr int kBridgeChunk = 256;
cudaError_t launch_bridge_merge(const int32_t* types, int64_t n, int64_t seq, int4* counts, const int32_t* grid_dev,
                                int n_images, int r, int64_t n_tokens, const void* image_tokens, const void* sentinels,
                                void* embeds, int row_vec, uint32_t* err, cudaStream_t s);
cudaError_t launch_image_visibility(const int32_t* types, int64_t batch, int64_t seq, void* mask, int elem_bytes,
                                    int4* counts, int32_t* span_first, int32_t* span_last, int32_t* span_of,
                                    uint32_t* err, cudaStream_t s);
// Norm operands of the first GEMM of a block: xw = bf16(x * w) and ss[p * parts] = sum_c x[p,c]^2
// (the other parts of a row are zero-filled); also clears zero_n counters like the kernels above.
cudaError_t launch_norm_prep(const void* x, const float* w, void* xw, float* ss, int parts, int64_t rows, int d,
                             cudaStream_t s, int* zero_ptr = nullptr, int zero_n = 0);

// ---------------------------------------------------------------------------- fp32 CUDA-core path
cudaError_t launch_gemm_f32(int epi, const float* a, const float* b, const float* b2, float* out, const float* resid,
                            int M, int n_out, int K, cudaStream_t s, const float* bias = nullptr);
cudaError_t launch_rope_apply_f32(float* qkv, const float* cos, const float* sin, int64_t P, int d, int n_heads,
                                  cudaStream_t s);
cudaError_t launch_attention_f32(const float* qkv, float* out, const int32_t* cu_dev, int n_images, int64_t P,
                                 int d, int n_heads, cudaStream_t s);
cudaError_t launch_gather_f32(const float* x, const int32_t* src, float* merged, int64_t n_tokens, int r2, int d,
                              cudaStream_t s);

}  // namespace dsv4v
