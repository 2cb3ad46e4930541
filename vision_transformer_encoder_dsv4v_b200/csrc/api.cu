// C ABI of the vision-tower forward: argument validation, workspace layout, GEMM planning,
// TMA descriptor construction and the launch sequence of each entry point.
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include <mutex>
#include <unordered_map>
#include <vector>

#include "dsv4v.h"
#include "common.cuh"
#include "internal.h"

namespace dsv4v {

// Device word in which kernels record the first bounded-wait timeout.
__device__ uint32_t g_dev_error;

namespace {

// ---------------------------------------------------------------------------- device info
struct DeviceInfo {
  int sms = 0;
  uint32_t* err = nullptr;
};

bool device_info(DeviceInfo& out) {
  static std::mutex mu;
  static std::unordered_map<int, DeviceInfo> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) {
    out = it->second;
    return true;
  }
  DeviceInfo info;
  if (cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return false;
  info.err = static_cast<uint32_t*>(p);
  cache[dev] = info;
  out = info;
  return true;
}

// SM count used for planning when no device can be queried (sizing only).
int planning_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
    return sms;
  cudaGetLastError();
  return 148;
}

// ---------------------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct MapKey {
  const void* ptr;
  int64_t rows, cols, ld;
  int box_rows;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && rows == o.rows && cols == o.cols && ld == o.ld && box_rows == o.box_rows;
  }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    size_t h = reinterpret_cast<size_t>(k.ptr);
    h ^= static_cast<size_t>(k.rows) * 0x9E3779B97F4A7C15ull;
    h ^= static_cast<size_t>(k.cols) * 0xC2B2AE3D27D4EB4Full + (h << 6);
    h ^= static_cast<size_t>(k.box_rows) * 0x165667B19E3779F9ull + (h >> 2);
    h ^= static_cast<size_t>(k.ld) * 0x27D4EB2F165667C5ull + (h << 3);
    return h;
  }
};

// bf16 row-major [rows, cols] matrix with row stride ld elements (0: cols; a multiple of 8),
// boxes of 64 columns (128 B, 128-byte swizzle) x box_rows rows; reads past the end of a row or
// of the matrix return zeros.  Descriptors depend only on these values, so they are cached per
// thread.
bool bf16_map(const void* ptr, int64_t rows, int64_t cols, int box_rows, CUtensorMap* out, int64_t ld = 0) {
  thread_local std::unordered_map<MapKey, CUtensorMap, MapKeyHash> cache;
  if (ld == 0) ld = cols;
  MapKey key{ptr, rows, cols, ld, box_rows};
  auto it = cache.find(key);
  if (it != cache.end()) {
    *out = it->second;
    return true;
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMap m;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  if (cache.size() > 4096) cache.clear();
  cache[key] = m;
  *out = m;
  return true;
}

// ---------------------------------------------------------------------------- validation
struct Shape {
  int D, H, hd, F, r, E, L;
  bool bf16;
  int64_t P, T;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dsv4v_status check_config(const dsv4v_config* c, Shape& s) {
  if (!c) return DSV4V_ERR_INVALID_ARG;
  if (c->vision_dim <= 0 || c->n_heads <= 0 || c->mlp_hidden <= 0 || c->downsample_ratio <= 0 || c->llm_dim <= 0 ||
      c->n_layers < 0 || !(c->eps >= 0.0f) || !(c->rope_theta > 0.0f))
    return DSV4V_ERR_INVALID_ARG;
  if (c->dtype != DSV4V_F32 && c->dtype != DSV4V_BF16) return DSV4V_ERR_INVALID_ARG;
  if (c->vision_dim % c->n_heads) return DSV4V_ERR_INVALID_ARG;
  s.D = c->vision_dim;
  s.H = c->n_heads;
  s.hd = s.D / s.H;
  s.F = c->mlp_hidden;
  s.r = c->downsample_ratio;
  s.E = c->llm_dim;
  s.L = c->n_layers;
  s.bf16 = c->dtype == DSV4V_BF16;
  if (s.hd % 4) return DSV4V_ERR_UNSUPPORTED;
  if (s.bf16) {
    if (s.hd != 64 || s.D % 128 || s.F % 128 || s.E % 128) return DSV4V_ERR_UNSUPPORTED;
  } else {
    if (s.hd > 64) return DSV4V_ERR_UNSUPPORTED;
  }
  return DSV4V_OK;
}

dsv4v_status check_batch(const dsv4v_batch* b, Shape& s) {
  if (!b || b->n_images < 1 || b->n_images > DSV4V_MAX_IMAGES) return DSV4V_ERR_INVALID_ARG;
  if (!b->grid_hw_host || !b->cu_patches_host || !b->grid_hw_dev || !b->cu_patches_dev) return DSV4V_ERR_INVALID_ARG;
  if (b->cu_patches_host[0] != 0) return DSV4V_ERR_INVALID_ARG;
  int64_t p = 0, t = 0;
  for (int i = 0; i < b->n_images; ++i) {
    const int64_t n_h = b->grid_hw_host[2 * i], n_w = b->grid_hw_host[2 * i + 1];
    if (n_h < 1 || n_w < 1) return DSV4V_ERR_INVALID_ARG;
    if (static_cast<int64_t>(b->cu_patches_host[i + 1]) - b->cu_patches_host[i] != n_h * n_w)
      return DSV4V_ERR_INVALID_ARG;
    p += n_h * n_w;
    t += ((n_h + s.r - 1) / s.r) * ((n_w + s.r - 1) / s.r);
    if (p > (1ll << 30)) return DSV4V_ERR_UNSUPPORTED;
  }
  s.P = p;
  s.T = t;
  return DSV4V_OK;
}

dsv4v_status check_all(const dsv4v_config* c, const dsv4v_batch* b, Shape& s) {
  dsv4v_status st = check_config(c, s);
  if (st != DSV4V_OK) return st;
  return check_batch(b, s);
}

// ---------------------------------------------------------------------------- chain plan
// Which launch sequence the bf16 blocks use: one kernel per GEMM, or the persistent chain kernel
// (chain.cu) that runs the output projection, SwiGLU, down projection and the next block's q|k|v
// projection in one launch per block.  Automatic choice: the chain for batches of at most
// kChainMaxRows patches (none at present: measured on B200, the chain does not yet beat one
// kernel per GEMM at 784 patches).
std::atomic<int> g_tower_path{DSV4V_PATH_AUTO};
constexpr int64_t kChainMaxRows = 0;
constexpr int kChainRingSlotsMax = 8;  // operand ring slots of the chain kernel (at most)

struct ChainStagePlan {
  int bn = 0, splits = 1, tiles_n = 0, kb = 0;
};
struct ChainPlan {
  bool use = false;
  int tiles_m = 0;
  ChainStagePlan st[4];  // output projection, SwiGLU, down projection, q|k|v projection
};
enum { CS_OUT = 0, CS_GATEUP = 1, CS_DOWN = 2, CS_QKV = 3 };

// Estimated cycles of one stage (fitted constants, B200): a 64-deep K block of a 128 x bn tile
// costs ~390 cycles at bn = 128 (the MMA instruction floor), ~478 at bn = 192 and ~574 at
// bn = 256 (the rate at which an SM takes in 48 KB of operands); tasks of one stage run in waves
// over the SMs; a split tile adds its partials' round trip through L2 and the epilogue ~8 cycles
// per column.
double chain_stage_cycles(int bn, int kb, int tasks, int splits, int sms) {
  const double kb_cyc = bn >= 256 ? 574.0 : (bn >= 192 ? 478.0 : 390.0);
  const int waves = (tasks + sms - 1) / sms;
  const int kb_per = (kb + splits - 1) / splits;
  double c = waves * kb_per * kb_cyc + 8.0 * bn;
  if (splits > 1) c += 1500.0 + (splits - 1) * 6.0 * bn;
  return c;
}

ChainStagePlan plan_chain_stage(int stage, const Shape& s, int tiles_m, int sms) {
  ChainStagePlan best;
  double best_c = 1e300;
  const int K = stage == CS_DOWN ? s.F : s.D;
  const int kb = (K + 63) / 64;
  const int n_cols = stage == CS_GATEUP ? s.F : s.D;
  // SwiGLU takes 256-column tiles (128 gate + 128 up): measured on B200 at 784 rows, two waves of
  // them finish ~8 us sooner than three waves of 128-column tiles.
  const int bns[2] = {256, 128};
  for (int bi = 0; bi < (stage == CS_QKV || stage == CS_GATEUP ? 1 : 2); ++bi) {
    const int bn = stage == CS_QKV ? 192 : bns[bi];
    const int cols = stage == CS_QKV ? 64 : (stage == CS_GATEUP ? bn / 2 : bn);
    if (n_cols % cols) continue;
    const int tiles_n = n_cols / cols;
    // SwiGLU and the q|k|v projection finish whole tiles; the residual GEMMs may split K.
    const int max_splits = (stage == CS_OUT || stage == CS_DOWN) ? 4 : 1;
    for (int sp = 1; sp <= max_splits && sp <= kb; ++sp) {
      const double c = chain_stage_cycles(bn, kb, tiles_m * tiles_n * sp, sp, sms);
      if (c < best_c - 1e-9) {
        best_c = c;
        best.bn = bn;
        best.splits = sp;
        best.tiles_n = tiles_n;
        best.kb = kb;
      }
    }
  }
  return best;
}

ChainPlan make_chain_plan(const Shape& s, int sms) {
  ChainPlan cp;
  if (!s.bf16 || s.P <= 0) return cp;
  const int path = g_tower_path.load();
  if (path == DSV4V_PATH_KERNELS || (path == DSV4V_PATH_AUTO && s.P > kChainMaxRows)) return cp;
  if (s.hd != 64 || s.D % 256 || s.F % 128) return cp;
  cp.tiles_m = static_cast<int>((s.P + 127) / 128);
  for (int st = 0; st < 4; ++st) cp.st[st] = plan_chain_stage(st, s, cp.tiles_m, sms);
  for (int st = 0; st < 4; ++st)
    if (cp.st[st].bn == 0) return ChainPlan{};
  cp.use = true;
  return cp;
}

// ---------------------------------------------------------------------------- workspace
struct Plans {
  GemmPlan qkv, out, gateup, down, align;
  ChainPlan chain;
};

Plans make_plans(const Shape& s, int sms) {
  Plans p;
  p.qkv = plan_gemm(EPI_QKV_ROPE, static_cast<int>(s.P), 3 * s.D, s.D, sms);
  p.out = plan_gemm(EPI_RESID, static_cast<int>(s.P), s.D, s.D, sms);
  p.gateup = plan_gemm(EPI_SWIGLU, static_cast<int>(s.P), s.F, s.D, sms);
  p.down = plan_gemm(EPI_RESID, static_cast<int>(s.P), s.D, s.F, sms);
  p.align = plan_gemm(EPI_STORE, static_cast<int>(s.T), s.E, s.r * s.r * s.D, sms);
  p.chain = make_chain_plan(s, sms);
  return p;
}

struct Layout {
  size_t cos, sin, y, qkv, attn, h, partials, counters, asrc, merged, ss1, ss2, total;
  size_t counters_bytes;
  int ss_parts;  // row stride of ss1 / ss2: the most N tiles a residual GEMM can have
  // chain kernel: fp32 split partials of each stage, and (inside the counters region, which the
  // first kernel of every call clears) per launch a ticket and per stage and row tile a
  // finished-tile counter, then per stage the split arrival counters
  size_t chain_partials[4];
  int chain_launches;   // launches the counters are laid out for
  int chain_ctr_off;    // int offset of the chain counters inside the counters region
  int chain_arr_off[4]; // int offsets of each stage's arrival counters
};

// Chain counters of launch `l`: [ticket][stage 0 done x tiles_m][stage 1 ...] ... [stage 3].
inline int chain_launch_ints(const ChainPlan& cp) { return 1 + 4 * cp.tiles_m; }

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Layout make_layout(const Shape& s, const Plans& pl) {
  Layout l{};
  const size_t es = s.bf16 ? 2 : 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off += up256(bytes);
    return at;
  };
  l.cos = take(static_cast<size_t>(s.P) * (s.hd / 2) * 4);
  l.sin = take(static_cast<size_t>(s.P) * (s.hd / 2) * 4);
  l.y = take(static_cast<size_t>(s.P) * s.D * es);
  l.qkv = take(static_cast<size_t>(s.P) * 3 * s.D * es);
  l.attn = take(static_cast<size_t>(s.P) * s.D * es);
  l.h = take(static_cast<size_t>(s.P) * s.F * es);
  size_t part = 0;
  int counters = 1;
  if (s.bf16) {
    const GemmPlan* all[5] = {&pl.qkv, &pl.out, &pl.gateup, &pl.down, &pl.align};
    for (const GemmPlan* g : all) {
      part = std::max(part, g->partial_bytes);
      counters = std::max(counters, g->counters);
    }
  }
  l.partials = take(part);
  int n_ints = counters;
  if (pl.chain.use) {
    const ChainPlan& cp = pl.chain;
    for (int st = 0; st < 4; ++st) {
      const ChainStagePlan& sp = cp.st[st];
      l.chain_partials[st] = take(sp.splits > 1 ? static_cast<size_t>(cp.tiles_m) * sp.tiles_n * (sp.splits - 1) *
                                                          128 * sp.bn * sizeof(float)
                                                    : 0);
    }
    l.chain_launches = std::max(2, s.L + 1);
    l.chain_ctr_off = counters;
    n_ints = counters + l.chain_launches * chain_launch_ints(cp);
    for (int st = 0; st < 4; ++st) {
      l.chain_arr_off[st] = n_ints;
      n_ints += cp.st[st].splits > 1 ? cp.tiles_m * cp.st[st].tiles_n : 0;
    }
  }
  l.counters_bytes = up256(static_cast<size_t>(n_ints) * sizeof(int));
  l.counters = take(l.counters_bytes);
  l.asrc = take(static_cast<size_t>(s.T) * s.r * s.r * 4);
  l.ss_parts = s.D / 64 > 0 ? s.D / 64 : 1;
  l.ss1 = take(s.bf16 ? static_cast<size_t>(s.P) * l.ss_parts * 4 : 0);
  l.ss2 = take(s.bf16 ? static_cast<size_t>(s.P) * l.ss_parts * 4 : 0);
  l.merged = take(static_cast<size_t>(s.T) * s.r * s.r * s.D * es);
  l.total = off;
  return l;
}

struct Ctx {
  Shape s;
  float eps, theta;
  Plans plans;
  Layout lay;
  DeviceInfo dev;
  uint8_t* ws;
  cudaStream_t stream;
  template <class T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

dsv4v_status prepare(const dsv4v_config* c, const dsv4v_batch* b, void* workspace, size_t ws_bytes, void* stream,
                     Ctx& ctx) {
  dsv4v_status st = check_all(c, b, ctx.s);
  if (st != DSV4V_OK) return st;
  if (!device_info(ctx.dev)) return DSV4V_ERR_CUDA;
  ctx.plans = make_plans(ctx.s, ctx.dev.sms);
  ctx.lay = make_layout(ctx.s, ctx.plans);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < ctx.lay.total)
    return DSV4V_ERR_WORKSPACE;
  ctx.eps = c->eps;
  ctx.theta = c->rope_theta;
  ctx.ws = static_cast<uint8_t*>(workspace);
  ctx.stream = static_cast<cudaStream_t>(stream);
  return DSV4V_OK;
}

dsv4v_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSV4V_OK : DSV4V_ERR_CUDA; }

#define DSV4V_TRY(expr)                           \
  do {                                            \
    dsv4v_status st_ = (expr);                    \
    if (st_ != DSV4V_OK) return st_;              \
  } while (0)

// ---------------------------------------------------------------------------- bf16 steps
// Folded-RMSNorm operands of one GEMM launch (see GemmArgs); all NULL / 0 = none.
struct NormFold {
  const float* ss = nullptr;  // consumer: partial sums of x^2 per row, `parts` of them at row stride `stride`
  int parts = 0;
  int stride = 0;
  void* xw_out = nullptr;     // producer: bf16(x * w) and its partial sums of x^2
  const float* xw_w = nullptr;
  float* ss_out = nullptr;
  int ss_parts = 0;
};

// Row strides of A and B when they are not K (0: K), and the STORE epilogue's bias.
struct GemmExtra {
  int64_t lda = 0, ldb = 0;
  const float* bias = nullptr;
  int clear_counters = 0;  // zero this many split-tile counters on the stream right before the launch
  // B (and B2) are the caller's weights, complete before the call: see GemmArgs::b_early.
  bool b_early = true;
  // Weights of the GEMM that follows, prefetched into L2 by this one (see GemmArgs).
  const void* l2_next[2] = {nullptr, nullptr};
  size_t l2_next_bytes[2] = {0, 0};
  // MN-major operands (STORE only, see GemmArgs::mn_major): a_mn, A is given as its stored
  // [K, M] matrix (row stride lda); b_mn, B as its stored [K, n_out] matrix (row stride ldb),
  // continued along K by b2 from K row kb_split * 64 on when b2 is set.
  bool a_mn = false, b_mn = false;
  int kb_split = 0;
};

GemmExtra prefetching(const void* w0, size_t bytes0, const void* w1 = nullptr, size_t bytes1 = 0) {
  GemmExtra ex;
  ex.l2_next[0] = w0;
  ex.l2_next_bytes[0] = w0 ? bytes0 : 0;
  ex.l2_next[1] = w1;
  ex.l2_next_bytes[1] = w1 ? bytes1 : 0;
  return ex;
}

dsv4v_status gemm_bf16(const Ctx& c, int epi, const GemmPlan& plan, const void* a, int64_t M, int K, const void* b,
                       const void* b2, int n_out, void* out, const void* resid, const float* cos = nullptr,
                       const float* sin = nullptr, const NormFold& nf = NormFold(), const GemmExtra& ex = GemmExtra()) {
  if (M == 0) return DSV4V_OK;
  const int box_b = (epi == EPI_SWIGLU || plan.pair) ? plan.bn / 2 : plan.bn;
  const bool b_split = ex.b_mn && b2 != nullptr;
  const int k_b1 = b_split ? ex.kb_split * 64 : K;  // K rows of B held by b
  CUtensorMap ta, tb, tb2, t_out, t_xw;
  const bool a_ok = ex.a_mn ? bf16_map(a, K, M, 64, &ta, ex.lda) : bf16_map(a, M, K, 128, &ta, ex.lda);
  const bool b_ok = ex.b_mn ? bf16_map(b, k_b1, n_out, 64, &tb, ex.ldb) : bf16_map(b, n_out, K, box_b, &tb, ex.ldb);
  const bool b2_ok = b_split ? bf16_map(b2, K - k_b1, n_out, 64, &tb2, ex.ldb)
                             : (epi != EPI_SWIGLU || bf16_map(b2, n_out, K, box_b, &tb2));
  if (!a_ok || !b_ok || !b2_ok || !bf16_map(out, M, n_out, 32, &t_out) ||
      (nf.xw_out && !bf16_map(nf.xw_out, M, n_out, 32, &t_xw)))
    return DSV4V_ERR_CUDA;
  GemmArgs g{};
  g.tm_out = &t_out;
  g.tm_xw = nf.xw_out ? &t_xw : nullptr;
  g.tm_a = &ta;
  g.tm_b = &tb;
  g.tm_b2 = (epi == EPI_SWIGLU || b_split) ? &tb2 : nullptr;
  g.mn_major = (ex.b_mn ? 1 : 0) | (ex.a_mn ? 2 : 0) | (b_split ? 4 : 0);
  g.kb_split = b_split ? ex.kb_split : 0;
  g.M = static_cast<int>(M);
  g.K = K;
  g.n_out = n_out;
  g.out = out;
  g.ldo = n_out;
  g.resid = resid;
  g.cos = cos;
  g.sin = sin;
  g.rot_cols = 2 * c.s.D;
  g.partials = c.at<float>(c.lay.partials);
  g.counters = c.at<int>(c.lay.counters);
  g.err = c.dev.err;
  g.norm_ss = nf.ss;
  g.norm_parts = nf.parts;
  g.norm_stride = nf.stride;
  g.norm_inv_d = 1.0f / static_cast<float>(c.s.D);
  g.norm_eps = c.eps;
  g.xw_out = nf.xw_out;
  g.xw_w = nf.xw_w;
  g.ss_out = nf.ss_out;
  g.ss_parts = nf.ss_parts;
  g.bias = ex.bias;
  g.b_early = ex.b_early;
  for (int r = 0; r < 2; ++r) {
    g.l2_next[r] = ex.l2_next[r];
    g.l2_next_bytes[r] = ex.l2_next_bytes[r];
  }
  if (ex.clear_counters > 0 &&
      cudaMemsetAsync(g.counters, 0, static_cast<size_t>(ex.clear_counters) * sizeof(int), c.stream) != cudaSuccess)
    return DSV4V_ERR_CUDA;
  return cuda_status(launch_gemm_tc(epi, plan, g, c.stream));
}

// Work items of the attention kernels: images longest first, per image its 128-row tiles in
// groups of `pair` (item_start, img_row0, img_len in that order).
void attention_schedule(const dsv4v_batch* b, int pair, int heads_per_item, AttnSchedule& sched) {
  const int n = b->n_images;
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  // Longest image first: its items cost the most (cost grows with the key count).
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
    return b->cu_patches_host[x + 1] - b->cu_patches_host[x] > b->cu_patches_host[y + 1] - b->cu_patches_host[y];
  });
  sched.n_images = n;
  sched.pair = pair;
  sched.split = 0;
  int items = 0;
  for (int k = 0; k < n; ++k) {
    const int i = order[k];
    const int len = b->cu_patches_host[i + 1] - b->cu_patches_host[i];
    sched.item_start[k] = items;
    sched.img_row0[k] = b->cu_patches_host[i];
    sched.img_len[k] = len;
    const int qt = (len + 127) / 128;
    items += ((qt + pair - 1) / pair) * heads_per_item;
  }
  sched.item_start[n] = items;
  sched.n_items = items;
}

dsv4v_status attention_bf16(const Ctx& c, const dsv4v_batch* b, const void* qkv, void* out, float* lse = nullptr) {
  CUtensorMap tm;
  if (!bf16_map(qkv, c.s.P, 3 * c.s.D, 128, &tm)) return DSV4V_ERR_CUDA;
  thread_local AttnSchedule sched;
  // Two query tiles per CTA halve the K/V traffic and keep two softmax warps on every SM
  // sub-partition; one per CTA when pairing would leave SMs idle.
  int paired = 0;
  for (int i = 0; i < b->n_images; ++i) {
    const int len = b->cu_patches_host[i + 1] - b->cu_patches_host[i];
    paired += ((len + 255) / 256) * c.s.H;
  }
  attention_schedule(b, paired >= c.dev.sms ? 2 : 1, c.s.H, sched);
  // Unpaired items (fewer than the SMs): both softmax warpgroups of a CTA work on its query tile,
  // each on every other key tile, so that each SM sub-partition runs two softmax warps.
  sched.split = sched.pair == 1 ? 1 : 0;
  return cuda_status(launch_attention_tc(&tm, sched, c.s.H, c.s.D, out, c.dev.err, c.stream, lse, c.s.P));
}

// One block on the bf16 path.  The two RMSNorms are folded into the GEMMs that consume them:
// the residual epilogue before each norm also writes xw = bf16(x * w) and the row partial sums
// of x^2, and the consuming GEMM (QKV, SwiGLU) reads xw and scales its rows by
// 1/sqrt(mean(x^2) + eps).  The first norm of a block with no residual GEMM before it comes from
// k_norm_prep.  next_norm_w: the norm1 weight of the following block, so that this block's last
// epilogue prepares it (NULL for the last block).
dsv4v_status record(void* const* ev, int kind, int which, cudaStream_t s) {
  if (!ev || !ev[kind * 2 + which]) return DSV4V_OK;
  cudaEvent_t e = static_cast<cudaEvent_t>(ev[kind * 2 + which]);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return DSV4V_ERR_CUDA;
  // Inside a stream capture an external record becomes an event-record node of the graph.
  return cuda_status(cap == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(e, s, cudaEventRecordExternal)
                                                          : cudaEventRecord(e, s));
}

dsv4v_status block_bf16(const Ctx& c, const dsv4v_batch* b, const dsv4v_block_weights* w, const float* cos,
                        const float* sin, void* x, bool first, const dsv4v_block_weights* next,
                        void* const* ev = nullptr) {
  const float* next_norm_w = next ? next->norm1_w : nullptr;
  // Each GEMM prefetches the weights of the next one into L2 (the block's weights come from HBM
  // once per step; the next GEMM then starts on L2 hits).
  const size_t dd = static_cast<size_t>(c.s.D) * c.s.D * 2, fd = static_cast<size_t>(c.s.F) * c.s.D * 2;
  const Shape& s = c.s;
  void* xw = c.at<void>(c.lay.y);
  void* qkv = c.at<void>(c.lay.qkv);
  void* attn = c.at<void>(c.lay.attn);
  void* h = c.at<void>(c.lay.h);
  float* ss1 = c.at<float>(c.lay.ss1);
  float* ss2 = c.at<float>(c.lay.ss2);
  if (first) {
    // The block's first kernel also clears the split-tile counters of its GEMMs.
    DSV4V_TRY(cuda_status(launch_norm_prep(x, w->norm1_w, xw, ss1, c.lay.ss_parts, s.P, s.D, c.stream,
                                           c.at<int>(c.lay.counters),
                                           static_cast<int>(c.lay.counters_bytes / sizeof(int)))));
  }
  NormFold q;
  q.ss = ss1;
  q.parts = first ? 1 : norm_parts_of(c.plans.down);  // the prep kernel puts the whole row sum in slot 0
  q.stride = c.lay.ss_parts;
  DSV4V_TRY(record(ev, DSV4V_PROFILE_QKV, 0, c.stream));
  DSV4V_TRY(gemm_bf16(c, EPI_QKV_ROPE, c.plans.qkv, xw, s.P, s.D, w->wqkv, nullptr, 3 * s.D, qkv, nullptr, cos,
                      sin, q, prefetching(w->wo, dd)));
  DSV4V_TRY(record(ev, DSV4V_PROFILE_QKV, 1, c.stream));
  DSV4V_TRY(record(ev, DSV4V_PROFILE_ATTENTION, 0, c.stream));
  DSV4V_TRY(attention_bf16(c, b, qkv, attn));
  DSV4V_TRY(record(ev, DSV4V_PROFILE_ATTENTION, 1, c.stream));
  NormFold o;
  o.xw_out = xw;
  o.xw_w = w->norm2_w;
  o.ss_out = ss2;
  o.ss_parts = c.lay.ss_parts;
  DSV4V_TRY(record(ev, DSV4V_PROFILE_OUT, 0, c.stream));
  DSV4V_TRY(gemm_bf16(c, EPI_RESID, c.plans.out, attn, s.P, s.D, w->wo, nullptr, s.D, x, x, nullptr, nullptr, o,
                      prefetching(w->w_gate, fd, w->w_up, fd)));
  DSV4V_TRY(record(ev, DSV4V_PROFILE_OUT, 1, c.stream));
  NormFold m;
  m.ss = ss2;
  m.parts = norm_parts_of(c.plans.out);
  m.stride = c.lay.ss_parts;
  DSV4V_TRY(record(ev, DSV4V_PROFILE_SWIGLU, 0, c.stream));
  DSV4V_TRY(gemm_bf16(c, EPI_SWIGLU, c.plans.gateup, xw, s.P, s.D, w->w_gate, w->w_up, s.F, h, nullptr, nullptr,
                      nullptr, m, prefetching(w->w_down, fd)));
  DSV4V_TRY(record(ev, DSV4V_PROFILE_SWIGLU, 1, c.stream));
  NormFold d;
  if (next_norm_w) {
    d.xw_out = xw;
    d.xw_w = next_norm_w;
    d.ss_out = ss1;
    d.ss_parts = c.lay.ss_parts;
  }
  DSV4V_TRY(record(ev, DSV4V_PROFILE_DOWN, 0, c.stream));
  DSV4V_TRY(gemm_bf16(c, EPI_RESID, c.plans.down, h, s.P, s.F, w->w_down, nullptr, s.D, x, x, nullptr, nullptr, d,
                      prefetching(next ? next->wqkv : nullptr, 3 * dd)));
  return record(ev, DSV4V_PROFILE_DOWN, 1, c.stream);
}

// ---------------------------------------------------------------------------- chain path
// Tensor maps of one chain launch, shared between stages that use the same tensor and box.
struct ChainBuilder {
  ChainParams p{};
  const void* key_ptr[kChainMaxMaps] = {};
  int key_box[kChainMaxMaps] = {};
  bool ok = true;
  int map(const void* ptr, int64_t rows, int64_t cols, int box) {
    for (int i = 0; i < p.n_maps; ++i)
      if (key_ptr[i] == ptr && key_box[i] == box) return i;
    if (p.n_maps >= kChainMaxMaps || !bf16_map(ptr, rows, cols, box, &p.maps[p.n_maps])) {
      ok = false;
      return 0;
    }
    key_ptr[p.n_maps] = ptr;
    key_box[p.n_maps] = box;
    return p.n_maps++;
  }
};

// One chain launch: the output projection, SwiGLU and down projection of block `cur` (NULL:
// none) followed by the q|k|v projection of block `next` (NULL: none).  `launch` selects this
// launch's ticket and row-tile counters.  next_norm1_w: the norm1 weight of `next`, which the
// down projection's epilogue prepares (NULL when `cur` is the last block); the q|k|v projection
// of a launch without `cur` takes its norm operand from k_norm_prep (whole row sum in slot 0).
dsv4v_status run_chain(const Ctx& c, int launch, const dsv4v_block_weights* cur, const dsv4v_block_weights* next,
                       const float* next_norm1_w, const float* cos, const float* sin, void* x) {
  const Shape& s = c.s;
  const ChainPlan& cp = c.plans.chain;
  if (launch >= c.lay.chain_launches) return DSV4V_ERR_UNSUPPORTED;
  void* xw = c.at<void>(c.lay.y);
  void* qkv = c.at<void>(c.lay.qkv);
  void* attn = c.at<void>(c.lay.attn);
  void* h = c.at<void>(c.lay.h);
  float* ss1 = c.at<float>(c.lay.ss1);
  float* ss2 = c.at<float>(c.lay.ss2);
  int* ctr = c.at<int>(c.lay.counters);
  int* base = ctr + c.lay.chain_ctr_off + launch * chain_launch_ints(cp);
  ChainBuilder b;
  ChainParams& p = b.p;
  p.ticket = base;
  p.err = c.dev.err;
  p.norm_inv_d = 1.0f / static_cast<float>(s.D);
  p.norm_eps = c.eps;
  int task = 0;
  auto stage = [&](int cs) -> ChainStage& {
    ChainStage& d = p.st[p.n_stages++];
    d = ChainStage{};
    const ChainStagePlan& sp = cp.st[cs];
    d.bn = sp.bn;
    d.kb_total = sp.kb;
    d.tiles_m = cp.tiles_m;
    d.tiles_n = sp.tiles_n;
    d.splits = sp.splits;
    d.task_base = task;
    task += d.tiles_m * d.tiles_n * d.splits;
    d.dep_stage = -1;
    d.map_b2 = -1;
    d.map_xw = -1;
    d.M = static_cast<int>(s.P);
    d.D = s.D;
    d.done = base + 1 + cs * cp.tiles_m;
    if (sp.splits > 1) {
      d.partials = c.at<float>(c.lay.chain_partials[cs]);
      d.arrivals = ctr + c.lay.chain_arr_off[cs];
    }
    return d;
  };
  if (cur) {
    ChainStage& o = stage(CS_OUT);
    o.epi = CHAIN_RESID;
    o.map_a = b.map(attn, s.P, s.D, 128);
    o.map_b = b.map(cur->wo, s.D, s.D, o.bn);
    o.map_out = b.map(x, s.P, s.D, 32);
    o.map_xw = b.map(xw, s.P, s.D, 32);
    o.resid = x;
    o.ldr = s.D;
    o.xw_w = cur->norm2_w;
    o.ss_out = ss2;
    o.ss_parts = c.lay.ss_parts;
    ChainStage& g = stage(CS_GATEUP);
    g.epi = CHAIN_SWIGLU;
    g.dep_stage = 0;
    g.dep_target = p.st[0].tiles_n;
    g.map_a = b.map(xw, s.P, s.D, 128);
    g.map_b = b.map(cur->w_gate, s.F, s.D, g.bn / 2);
    g.map_b2 = b.map(cur->w_up, s.F, s.D, g.bn / 2);
    g.map_out = b.map(h, s.P, s.F, 32);
    g.norm_ss = ss2;
    g.norm_parts = p.st[0].tiles_n;
    g.norm_stride = c.lay.ss_parts;
    ChainStage& dn = stage(CS_DOWN);
    dn.epi = CHAIN_RESID;
    dn.dep_stage = 1;
    dn.dep_target = p.st[1].tiles_n;
    dn.map_a = b.map(h, s.P, s.F, 128);
    dn.map_b = b.map(cur->w_down, s.D, s.F, dn.bn);
    dn.map_out = b.map(x, s.P, s.D, 32);
    dn.resid = x;
    dn.ldr = s.D;
    if (next_norm1_w) {
      dn.map_xw = b.map(xw, s.P, s.D, 32);
      dn.xw_w = next_norm1_w;
      dn.ss_out = ss1;
      dn.ss_parts = c.lay.ss_parts;
    }
  }
  if (next) {
    ChainStage& q = stage(CS_QKV);
    q.epi = CHAIN_QKV_HEADS;
    q.dep_stage = cur ? 2 : -1;
    q.dep_target = cur ? p.st[2].tiles_n : 0;
    q.map_a = b.map(xw, s.P, s.D, 128);
    q.map_b = b.map(next->wqkv, 3 * s.D, s.D, 64);
    q.map_out = b.map(qkv, s.P, 3 * s.D, 32);
    q.cos = cos;
    q.sin = sin;
    q.norm_ss = ss1;
    q.norm_parts = cur ? p.st[2].tiles_n : 1;
    q.norm_stride = c.lay.ss_parts;
  }
  if (!b.ok) return DSV4V_ERR_CUDA;
  p.total_tasks = task;
  // Ring slots as large as the launch's largest stage (A + B tile of one K block), as many as fit.
  int stage_bytes = 0;
  for (int i = 0; i < p.n_stages; ++i) stage_bytes = std::max(stage_bytes, 128 * 64 * 2 + p.st[i].bn * 128);
  p.slot_bytes = (stage_bytes + 8191) / 8192 * 8192;
  p.ring_slots = std::min(kChainRingSlotsMax, chain_ring_bytes() / p.slot_bytes);
  return cuda_status(launch_chain(p, c.dev.sms, c.stream));
}

// Blocks [0, L) on the chain path: the first norm operand, layer 0's q|k|v projection, then per
// layer attention and one chain launch (layer l's remaining GEMMs and layer l + 1's q|k|v).
// The first kernel clears every counter of the call.  ev: DSV4V_PROFILE_* event pairs per layer.
dsv4v_status blocks_chain(const Ctx& c, const dsv4v_batch* b, const dsv4v_block_weights* layers, int L,
                          const float* cos, const float* sin, void* x, void* const* ev) {
  const Shape& s = c.s;
  DSV4V_TRY(cuda_status(launch_norm_prep(x, layers[0].norm1_w, c.at<void>(c.lay.y), c.at<float>(c.lay.ss1),
                                         c.lay.ss_parts, s.P, s.D, c.stream, c.at<int>(c.lay.counters),
                                         static_cast<int>(c.lay.counters_bytes / sizeof(int)))));
  DSV4V_TRY(run_chain(c, 0, nullptr, &layers[0], nullptr, cos, sin, x));
  for (int l = 0; l < L; ++l) {
    void* const* e = ev ? ev + static_cast<size_t>(l) * DSV4V_PROFILE_KINDS * 2 : nullptr;
    DSV4V_TRY(record(e, DSV4V_PROFILE_ATTENTION, 0, c.stream));
    DSV4V_TRY(attention_bf16(c, b, c.at<void>(c.lay.qkv), c.at<void>(c.lay.attn)));
    DSV4V_TRY(record(e, DSV4V_PROFILE_ATTENTION, 1, c.stream));
    DSV4V_TRY(record(e, DSV4V_PROFILE_CHAIN, 0, c.stream));
    DSV4V_TRY(run_chain(c, l + 1, &layers[l], l + 1 < L ? &layers[l + 1] : nullptr,
                        l + 1 < L ? layers[l + 1].norm1_w : nullptr, cos, sin, x));
    DSV4V_TRY(record(e, DSV4V_PROFILE_CHAIN, 1, c.stream));
  }
  return DSV4V_OK;
}

// ---------------------------------------------------------------------------- fp32 steps
dsv4v_status block_f32(const Ctx& c, const dsv4v_batch* b, const dsv4v_block_weights* w, const float* cos,
                       const float* sin, void* xv) {
  const Shape& s = c.s;
  float* x = static_cast<float*>(xv);
  float* y = c.at<float>(c.lay.y);
  float* qkv = c.at<float>(c.lay.qkv);
  float* attn = c.at<float>(c.lay.attn);
  float* h = c.at<float>(c.lay.h);
  const int M = static_cast<int>(s.P);
  DSV4V_TRY(cuda_status(launch_rmsnorm(false, x, w->norm1_w, y, s.P, s.D, c.eps, c.stream)));
  DSV4V_TRY(cuda_status(launch_gemm_f32(EPI_STORE, y, static_cast<const float*>(w->wqkv), nullptr, qkv, nullptr, M,
                                        3 * s.D, s.D, c.stream)));
  DSV4V_TRY(cuda_status(launch_rope_apply_f32(qkv, cos, sin, s.P, s.D, s.H, c.stream)));
  DSV4V_TRY(cuda_status(launch_attention_f32(qkv, attn, b->cu_patches_dev, b->n_images, s.P, s.D, s.H, c.stream)));
  DSV4V_TRY(cuda_status(launch_gemm_f32(EPI_RESID, attn, static_cast<const float*>(w->wo), nullptr, x, x, M, s.D, s.D,
                                        c.stream)));
  DSV4V_TRY(cuda_status(launch_rmsnorm(false, x, w->norm2_w, y, s.P, s.D, c.eps, c.stream)));
  DSV4V_TRY(cuda_status(launch_gemm_f32(EPI_SWIGLU, y, static_cast<const float*>(w->w_gate),
                                        static_cast<const float*>(w->w_up), h, nullptr, M, s.F, s.D, c.stream)));
  return cuda_status(launch_gemm_f32(EPI_RESID, h, static_cast<const float*>(w->w_down), nullptr, x, x, M, s.D, s.F,
                                     c.stream));
}

bool weights_ok(const dsv4v_block_weights* w) {
  return w && w->norm1_w && w->norm2_w && w->wqkv && w->wo && w->w_gate && w->w_up && w->w_down &&
         aligned16(w->norm1_w) && aligned16(w->norm2_w) && aligned16(w->wqkv) && aligned16(w->wo) &&
         aligned16(w->w_gate) && aligned16(w->w_up) && aligned16(w->w_down);
}

dsv4v_status reset_counters(const Ctx& c) {
  if (!c.s.bf16) return DSV4V_OK;
  return cuda_status(launch_zero_counters(c.at<int>(c.lay.counters), static_cast<int>(c.lay.counters_bytes / sizeof(int)),
                                          c.stream));
}

dsv4v_status rope_table(const Ctx& c, const dsv4v_batch* b, float* cos, float* sin) {
  return cuda_status(launch_rope_table(b->cu_patches_dev, b->grid_hw_dev, b->n_images, c.s.P, c.s.hd / 2, c.theta,
                                       cos, sin, c.stream, c.s.bf16 ? c.at<int>(c.lay.counters) : nullptr,
                                       c.s.bf16 ? static_cast<int>(c.lay.counters_bytes / sizeof(int)) : 0));
}

// Validation-only context for component calls that take a row count instead of a batch.
dsv4v_status prepare_rows(const dsv4v_config* cfg, int64_t rows, void* workspace, size_t ws_bytes, void* stream,
                          bool need_ws, Ctx& ctx) {
  DSV4V_TRY(check_config(cfg, ctx.s));
  if (rows < 0 || rows > (1ll << 30)) return DSV4V_ERR_INVALID_ARG;
  ctx.s.P = rows;
  ctx.s.T = 0;
  if (!device_info(ctx.dev)) return DSV4V_ERR_CUDA;
  ctx.plans = make_plans(ctx.s, ctx.dev.sms);
  ctx.lay = make_layout(ctx.s, ctx.plans);
  ctx.eps = cfg->eps;
  ctx.theta = cfg->rope_theta;
  ctx.stream = static_cast<cudaStream_t>(stream);
  ctx.ws = static_cast<uint8_t*>(workspace);
  if (need_ws && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < ctx.lay.total))
    return DSV4V_ERR_WORKSPACE;
  return DSV4V_OK;
}

}  // namespace

// Residual GEMM x <- x + a . w^T on the bf16 path with split-tile scratch supplied by the caller
// (partials: partial_cap bytes, counters: counter_cap ints).  Used by the entry point whose
// scratch is a static device array: that array keeps the last call's contents, so the counters
// the plan uses are cleared on the stream, but only once every argument and the plan have been
// accepted (a rejected call enqueues nothing).
dsv4v_status linear_residual_with_scratch(const dsv4v_config* cfg, int64_t rows, int k, const void* a,
                                          const void* w, void* x, float* partials, size_t partial_cap,
                                          int* counters, int counter_cap, void* stream) {
  Ctx c;
  DSV4V_TRY(check_config(cfg, c.s));
  if (!c.s.bf16) return DSV4V_ERR_UNSUPPORTED;
  if (rows < 0 || rows > (1ll << 30) || !a || !w || !x || !aligned16(a) || !aligned16(w) || !aligned16(x))
    return DSV4V_ERR_INVALID_ARG;
  if (k != c.s.D && k != c.s.F) return DSV4V_ERR_INVALID_ARG;
  if (rows == 0) return DSV4V_OK;
  if (!device_info(c.dev)) return DSV4V_ERR_CUDA;
  const GemmPlan plan = plan_gemm(EPI_RESID, static_cast<int>(rows), c.s.D, k, c.dev.sms, partial_cap);
  if (plan.bn == 0) return DSV4V_ERR_UNSUPPORTED;
  if (plan.partial_bytes > partial_cap || static_cast<size_t>(plan.counters) > static_cast<size_t>(counter_cap))
    return DSV4V_ERR_UNSUPPORTED;
  c.s.P = rows;
  c.s.T = 0;
  c.eps = cfg->eps;
  c.theta = cfg->rope_theta;
  c.stream = static_cast<cudaStream_t>(stream);
  // gemm_bf16 addresses scratch as offsets from c.ws: point it at the partials, counters follow.
  c.ws = reinterpret_cast<uint8_t*>(partials);
  c.lay = Layout{};
  c.lay.partials = 0;
  c.lay.counters = static_cast<size_t>(reinterpret_cast<uint8_t*>(counters) - reinterpret_cast<uint8_t*>(partials));
  GemmExtra ex;
  ex.clear_counters = plan.counters;
  return gemm_bf16(c, EPI_RESID, plan, a, rows, k, w, nullptr, c.s.D, x, x, nullptr, nullptr, NormFold(), ex);
}

// ----------------------------------------------------------------------------- graph replay
// A step of the 28x28 tower is ~170 launches of ~11 us each, so launching them one by one from
// the host costs a few percent against replaying them as one CUDA graph.  The step entry points
// therefore keep a small per-thread cache of graph executables (like the tensor-map cache)
// keyed by every argument that shapes their launches (the config, the batch's host arrays and
// device pointers, the weight, buffer and workspace pointers, the launch-sequence setting, the
// device).  The first call with a key runs eagerly (it also warms the plan and descriptor
// caches); the second captures the launches on the caller's stream (thread-local capture) and
// replays the instantiated graph, as do all later calls.  Calls on the legacy default stream,
// or on a stream that is already being captured (the caller's own graph), always launch
// directly.  A capture or instantiation that fails leaves that key on direct launches.
struct GraphEntry {
  std::vector<uint64_t> key;
  cudaGraphExec_t exec = nullptr;
  int state = 0;  // 1: seen once, 2: graph ready, -1: direct launches only
  uint64_t last_use = 0;
};

thread_local std::vector<GraphEntry> g_graphs;
thread_local uint64_t g_graph_clock = 0;
std::atomic<int> g_graph_replay{1};
constexpr size_t kMaxGraphs = 16;

struct KeyBuilder {
  std::vector<uint64_t> k;
  void u(uint64_t v) { k.push_back(v); }
  void p(const void* ptr) { k.push_back(reinterpret_cast<uint64_t>(ptr)); }
  void bytes(const void* src, size_t n) {
    const uint8_t* b = static_cast<const uint8_t*>(src);
    for (size_t i = 0; i < n; i += 8) {
      uint64_t v = 0;
      memcpy(&v, b + i, std::min<size_t>(8, n - i));
      k.push_back(v);
    }
  }
};

// Key prefix shared by the step entry points: which call, the device, the setting, the config
// and the batch (host values and device pointers).
KeyBuilder step_key(int call, const dsv4v_config* cfg, const dsv4v_batch* batch) {
  KeyBuilder kb;
  int dev = -1;
  cudaGetDevice(&dev);
  kb.u(static_cast<uint64_t>(call));
  kb.u(static_cast<uint64_t>(dev));
  kb.u(static_cast<uint64_t>(g_tower_path.load()));
  kb.bytes(cfg, sizeof(*cfg));
  kb.u(static_cast<uint64_t>(batch->n_images));
  kb.p(batch->grid_hw_dev);
  kb.p(batch->cu_patches_dev);
  kb.bytes(batch->grid_hw_host, sizeof(int32_t) * 2 * static_cast<size_t>(batch->n_images));
  kb.bytes(batch->cu_patches_host, sizeof(int32_t) * (static_cast<size_t>(batch->n_images) + 1));
  return kb;
}

template <class Run>
dsv4v_status with_graph(KeyBuilder&& kb, void* stream, Run&& run) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!g_graph_replay.load() || s == nullptr || s == cudaStreamLegacy || s == cudaStreamPerThread) return run();
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return run();
  }
  if (cs != cudaStreamCaptureStatusNone) return run();
  GraphEntry* e = nullptr;
  for (auto& g : g_graphs)
    if (g.key == kb.k) {
      e = &g;
      break;
    }
  if (e == nullptr) {
    if (g_graphs.size() >= kMaxGraphs) {
      // evict the least recently used entry (an executable still in flight is freed when it
      // completes)
      auto lru = std::min_element(g_graphs.begin(), g_graphs.end(),
                                  [](const GraphEntry& a, const GraphEntry& b) { return a.last_use < b.last_use; });
      if (lru->exec) cudaGraphExecDestroy(lru->exec);
      g_graphs.erase(lru);
    }
    g_graphs.push_back(GraphEntry{std::move(kb.k), nullptr, 1, ++g_graph_clock});
    return run();
  }
  e->last_use = ++g_graph_clock;
  if (e->state == 2) return cuda_status(cudaGraphLaunch(e->exec, s));
  if (e->state < 0) return run();
  // Second call with this key: capture it.
  if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    e->state = -1;
    return run();
  }
  const dsv4v_status st = run();
  cudaGraph_t graph = nullptr;
  const cudaError_t end = cudaStreamEndCapture(s, &graph);
  cudaGraphExec_t exec = nullptr;
  cudaError_t inst = cudaErrorUnknown;
  if (st == DSV4V_OK && end == cudaSuccess && graph != nullptr) inst = cudaGraphInstantiate(&exec, graph, 0);
  if (graph) cudaGraphDestroy(graph);
  if (inst != cudaSuccess) {
    // nothing of the captured call ran: run it directly
    cudaGetLastError();
    e->state = -1;
    return st == DSV4V_OK ? run() : st;
  }
  e->exec = exec;
  e->state = 2;
  return cuda_status(cudaGraphLaunch(exec, s));
}

}  // namespace dsv4v

using namespace dsv4v;

extern "C" {

void dsv4v_set_graph_replay(int enable) { g_graph_replay.store(enable ? 1 : 0); }

void dsv4v_release_graphs(void) {
  for (auto& g : g_graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  g_graphs.clear();
}

const char* dsv4v_status_string(dsv4v_status s) {
  switch (s) {
    case DSV4V_OK: return "ok";
    case DSV4V_ERR_INVALID_ARG: return "invalid argument";
    case DSV4V_ERR_UNSUPPORTED: return "unsupported shape";
    case DSV4V_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DSV4V_ERR_CUDA: return "CUDA error";
    case DSV4V_ERR_TIMEOUT: return "device-side check failed (wait timed out)";
    case DSV4V_ERR_LAYOUT: return "pseudo-token types do not fit the images";
  }
  return "unknown status";
}

int dsv4v_step_launches(const dsv4v_config* cfg, const dsv4v_batch* batch, int final_norm, int aligner) {
  Shape s;
  if (check_all(cfg, batch, s) != DSV4V_OK) return -1;
  const Plans pl = make_plans(s, planning_sms());
  int n = 1;  // rotary table
  if (s.L > 0) {
    if (s.bf16 && pl.chain.use) n += 2 + 2 * s.L;  // first norm operand, layer 0's q|k|v, attention + chain per layer
    else if (s.bf16) n += 1 + 5 * s.L;             // first norm operand, 4 GEMMs + attention per layer
    else n += 8 * s.L;                              // fp32: 2 norms, 4 GEMMs, rotation, attention per layer
  }
  if (final_norm) n += 1;
  if (aligner) n += 3;  // window index, merged rows, GEMM
  return n;
}

dsv4v_status dsv4v_set_tower_path(int path) {
  if (path != DSV4V_PATH_AUTO && path != DSV4V_PATH_KERNELS && path != DSV4V_PATH_CHAIN)
    return DSV4V_ERR_INVALID_ARG;
  g_tower_path.store(path);
  return DSV4V_OK;
}

int dsv4v_tower_path(const dsv4v_config* cfg, const dsv4v_batch* batch) {
  Shape s;
  if (check_all(cfg, batch, s) != DSV4V_OK) return -1;
  return make_chain_plan(s, planning_sms()).use ? DSV4V_PATH_CHAIN : DSV4V_PATH_KERNELS;
}

size_t dsv4v_workspace_size(const dsv4v_config* cfg, const dsv4v_batch* batch) {
  Shape s;
  if (check_all(cfg, batch, s) != DSV4V_OK) return 0;
  return make_layout(s, make_plans(s, planning_sms())).total;
}

int64_t dsv4v_aligner_tokens(const dsv4v_config* cfg, const dsv4v_batch* batch) {
  Shape s;
  if (check_all(cfg, batch, s) != DSV4V_OK) return -1;
  return s.T;
}

dsv4v_status dsv4v_rope2d_table(const dsv4v_config* cfg, const dsv4v_batch* batch, float* cos_out, float* sin_out,
                                void* stream) {
  Shape s;
  DSV4V_TRY(check_all(cfg, batch, s));
  if (!cos_out || !sin_out) return DSV4V_ERR_INVALID_ARG;
  return cuda_status(launch_rope_table(batch->cu_patches_dev, batch->grid_hw_dev, batch->n_images, s.P, s.hd / 2,
                                       cfg->rope_theta, cos_out, sin_out, static_cast<cudaStream_t>(stream)));
}

dsv4v_status dsv4v_block_forward(const dsv4v_config* cfg, const dsv4v_batch* batch, const dsv4v_block_weights* w,
                                 const float* cos, const float* sin, void* x_inout, void* workspace, size_t ws_bytes,
                                 void* stream) {
  Ctx c;
  DSV4V_TRY(prepare(cfg, batch, workspace, ws_bytes, stream, c));
  if (!weights_ok(w) || !cos || !sin || !x_inout || !aligned16(x_inout) || !aligned16(cos) || !aligned16(sin))
    return DSV4V_ERR_INVALID_ARG;
  if (c.s.bf16 && c.plans.chain.use) return blocks_chain(c, batch, w, 1, cos, sin, x_inout, nullptr);
  return c.s.bf16 ? block_bf16(c, batch, w, cos, sin, x_inout, true, nullptr)
                   : block_f32(c, batch, w, cos, sin, x_inout);
}

static dsv4v_status tower_impl(const dsv4v_config* cfg, const dsv4v_batch* batch, const dsv4v_block_weights* layers,
                               const float* final_norm_w, void* x_inout, void* workspace, size_t ws_bytes,
                               void* stream, void* const* events) {
  Ctx c;
  DSV4V_TRY(prepare(cfg, batch, workspace, ws_bytes, stream, c));
  if (!x_inout || !aligned16(x_inout) || (c.s.L > 0 && !layers)) return DSV4V_ERR_INVALID_ARG;
  for (int l = 0; l < c.s.L; ++l)
    if (!weights_ok(&layers[l])) return DSV4V_ERR_INVALID_ARG;
  if (final_norm_w && !aligned16(final_norm_w)) return DSV4V_ERR_INVALID_ARG;
  float* cos = c.at<float>(c.lay.cos);
  float* sin = c.at<float>(c.lay.sin);
  DSV4V_TRY(rope_table(c, batch, cos, sin));
  if (c.s.bf16 && c.plans.chain.use && c.s.L > 0) {
    DSV4V_TRY(blocks_chain(c, batch, layers, c.s.L, cos, sin, x_inout, events));
  } else {
    for (int l = 0; l < c.s.L; ++l)
      DSV4V_TRY(c.s.bf16 ? block_bf16(c, batch, &layers[l], cos, sin, x_inout, l == 0,
                                      l + 1 < c.s.L ? &layers[l + 1] : nullptr,
                                      events ? events + static_cast<size_t>(l) * DSV4V_PROFILE_KINDS * 2 : nullptr)
                         : block_f32(c, batch, &layers[l], cos, sin, x_inout));
  }
  if (final_norm_w)
    DSV4V_TRY(cuda_status(launch_rmsnorm(c.s.bf16, x_inout, final_norm_w, x_inout, c.s.P, c.s.D, c.eps, c.stream)));
  return DSV4V_OK;
}

dsv4v_status dsv4v_tower_forward(const dsv4v_config* cfg, const dsv4v_batch* batch, const dsv4v_block_weights* layers,
                                 const float* final_norm_w, void* x_inout, void* workspace, size_t ws_bytes,
                                 void* stream) {
  auto run = [&] { return tower_impl(cfg, batch, layers, final_norm_w, x_inout, workspace, ws_bytes, stream, nullptr); };
  Shape sh;
  if (check_all(cfg, batch, sh) != DSV4V_OK || (cfg->n_layers > 0 && !layers)) return run();
  KeyBuilder kb = step_key(1, cfg, batch);
  kb.bytes(layers, sizeof(dsv4v_block_weights) * static_cast<size_t>(cfg->n_layers));
  kb.p(final_norm_w);
  kb.p(x_inout);
  kb.p(workspace);
  kb.u(ws_bytes);
  return with_graph(std::move(kb), stream, run);
}

dsv4v_status dsv4v_tower_forward_profiled(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                          const dsv4v_block_weights* layers, const float* final_norm_w,
                                          void* x_inout, void* workspace, size_t ws_bytes, void* stream,
                                          void* const* events) {
  return tower_impl(cfg, batch, layers, final_norm_w, x_inout, workspace, ws_bytes, stream, events);
}

static dsv4v_status aligner_impl(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* x,
                                 const void* w_align, void* out, void* workspace, size_t ws_bytes, void* stream) {
  Ctx c;
  DSV4V_TRY(prepare(cfg, batch, workspace, ws_bytes, stream, c));
  if (!x || !w_align || !out || !aligned16(x) || !aligned16(w_align) || !aligned16(out)) return DSV4V_ERR_INVALID_ARG;
  const Shape& s = c.s;
  int32_t* src = c.at<int32_t>(c.lay.asrc);
  DSV4V_TRY(cuda_status(launch_aligner_index(batch->cu_patches_dev, batch->grid_hw_dev, batch->n_images, s.r, s.T,
                                             src, c.stream, s.bf16 ? c.at<int>(c.lay.counters) : nullptr,
                                             s.bf16 ? static_cast<int>(c.lay.counters_bytes / sizeof(int)) : 0)));
  const int K = s.r * s.r * s.D;
  if (s.bf16) {
    // Materialise the merged window rows, then a TMA GEMM (the weights stream once; the rows
    // are a few MB).  Gathering the rows inside the GEMM with TMA tile::gather4 (four source rows
    // per copy) measured 2.3x slower on B200: 53 us against 5 + 23 us.
    void* merged = c.at<uint8_t>(c.lay.merged);
    DSV4V_TRY(cuda_status(launch_merge_rows_bf16(x, src, merged, s.T, s.r * s.r, s.D, c.stream)));
    return gemm_bf16(c, EPI_STORE, c.plans.align, merged, s.T, K, w_align, nullptr, s.E, out, nullptr);
  }
  float* merged = c.at<float>(c.lay.merged);
  DSV4V_TRY(cuda_status(launch_gather_f32(static_cast<const float*>(x), src, merged, s.T, s.r * s.r, s.D, c.stream)));
  return cuda_status(launch_gemm_f32(EPI_STORE, merged, static_cast<const float*>(w_align), nullptr,
                                     static_cast<float*>(out), nullptr, static_cast<int>(s.T), s.E, K, c.stream));
}

dsv4v_status dsv4v_aligner_forward(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* x,
                                   const void* w_align, void* out, int32_t* cu_tokens_host, void* workspace,
                                   size_t ws_bytes, void* stream) {
  Shape sh;
  if (check_all(cfg, batch, sh) != DSV4V_OK) return aligner_impl(cfg, batch, x, w_align, out, workspace, ws_bytes, stream);
  if (cu_tokens_host) {
    // host output: written on every call, replayed or not
    int64_t t = 0;
    cu_tokens_host[0] = 0;
    for (int i = 0; i < batch->n_images; ++i) {
      const int n_h = batch->grid_hw_host[2 * i], n_w = batch->grid_hw_host[2 * i + 1];
      t += static_cast<int64_t>((n_h + sh.r - 1) / sh.r) * ((n_w + sh.r - 1) / sh.r);
      cu_tokens_host[i + 1] = static_cast<int32_t>(t);
    }
  }
  KeyBuilder kb = step_key(2, cfg, batch);
  kb.p(x);
  kb.p(w_align);
  kb.p(out);
  kb.p(workspace);
  kb.u(ws_bytes);
  return with_graph(std::move(kb), stream,
                    [&] { return aligner_impl(cfg, batch, x, w_align, out, workspace, ws_bytes, stream); });
}

// Scratch of the PatchMerger projector: window index [T, r^2] int32, merged rows and hidden rows
// [T, r^2 D] in the activation dtype.
namespace {
struct MergerLayout {
  GemmPlan p1, p2;  // Linear 1 (GELU epilogue) and Linear 2 (bias store)
  size_t src, merged, hidden, partials, counters, counters_bytes, total;
};
MergerLayout merger_layout(const Shape& s, int sms) {
  MergerLayout l{};
  const size_t es = s.bf16 ? 2 : 4;
  const size_t rows = static_cast<size_t>(s.T) * s.r * s.r;
  const int K = s.r * s.r * s.D;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += up256(bytes);
    return at;
  };
  l.src = take(rows * 4);
  l.merged = take(rows * s.D * es);
  l.hidden = take(rows * s.D * es);
  size_t part = 0;
  int counters = 1;
  if (s.bf16 && s.T > 0) {
    l.p1 = plan_gemm(EPI_GELU, static_cast<int>(s.T), K, K, sms);
    l.p2 = plan_gemm(EPI_STORE, static_cast<int>(s.T), s.E, K, sms);
    part = std::max(l.p1.partial_bytes, l.p2.partial_bytes);
    counters = std::max(counters, std::max(l.p1.counters, l.p2.counters));
  }
  l.partials = take(part);
  l.counters_bytes = up256(static_cast<size_t>(counters) * sizeof(int));
  l.counters = take(l.counters_bytes);
  l.total = off;
  return l;
}
}  // namespace

size_t dsv4v_patch_merger_workspace_size(const dsv4v_config* cfg, const dsv4v_batch* batch) {
  Shape s;
  if (check_all(cfg, batch, s) != DSV4V_OK) return 0;
  return merger_layout(s, planning_sms()).total;
}

dsv4v_status dsv4v_patch_merger_forward(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* x,
                                        const float* ln_w, const float* ln_b, const void* w1, const float* b1,
                                        const void* w2, const float* b2, void* out, void* workspace, size_t ws_bytes,
                                        void* stream) {
  Ctx c;
  DSV4V_TRY(check_all(cfg, batch, c.s));
  if (!device_info(c.dev)) return DSV4V_ERR_CUDA;
  const Shape& s = c.s;
  for (const void* ptr : {x, static_cast<const void*>(ln_w), static_cast<const void*>(ln_b), w1,
                          static_cast<const void*>(b1), w2, static_cast<const void*>(b2), static_cast<const void*>(out)})
    if (!ptr || !aligned16(ptr)) return DSV4V_ERR_INVALID_ARG;
  const MergerLayout l = merger_layout(s, c.dev.sms);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < l.total) return DSV4V_ERR_WORKSPACE;
  c.stream = static_cast<cudaStream_t>(stream);
  c.eps = cfg->eps;
  c.ws = static_cast<uint8_t*>(workspace);
  c.lay = Layout{};
  c.lay.partials = l.partials;  // split-tile scratch of the two GEMMs
  c.lay.counters = l.counters;
  c.lay.counters_bytes = l.counters_bytes;
  if (s.T == 0) return DSV4V_OK;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* src = reinterpret_cast<int32_t*>(ws + l.src);
  void* merged = ws + l.merged;
  void* hidden = ws + l.hidden;
  const int r2 = s.r * s.r, K = r2 * s.D;
  DSV4V_TRY(cuda_status(launch_aligner_index(batch->cu_patches_dev, batch->grid_hw_dev, batch->n_images, s.r, s.T, src,
                                             c.stream)));
  DSV4V_TRY(cuda_status(launch_ln_merge(s.bf16, x, src, ln_w, ln_b, cfg->eps, merged, s.T, r2, s.D, c.stream)));
  if (!s.bf16) {
    DSV4V_TRY(cuda_status(launch_gemm_f32(EPI_GELU, static_cast<const float*>(merged), static_cast<const float*>(w1),
                                          nullptr, static_cast<float*>(hidden), nullptr, static_cast<int>(s.T), K, K,
                                          c.stream, b1)));
    return cuda_status(launch_gemm_f32(EPI_STORE, static_cast<const float*>(hidden), static_cast<const float*>(w2),
                                       nullptr, static_cast<float*>(out), nullptr, static_cast<int>(s.T), s.E, K,
                                       c.stream, b2));
  }
  const GemmPlan& p1 = l.p1;
  const GemmPlan& p2 = l.p2;
  if (p1.bn == 0 || p2.bn == 0) return DSV4V_ERR_UNSUPPORTED;
  DSV4V_TRY(reset_counters(c));  // the finishers of each GEMM leave the counters at zero again
  GemmExtra e1, e2;
  e1.bias = b1;
  e2.bias = b2;
  DSV4V_TRY(gemm_bf16(c, EPI_GELU, p1, merged, s.T, K, w1, nullptr, K, hidden, nullptr, nullptr, nullptr, NormFold(),
                      e1));
  return gemm_bf16(c, EPI_STORE, p2, hidden, s.T, K, w2, nullptr, s.E, out, nullptr, nullptr, nullptr, NormFold(), e2);
}

dsv4v_status dsv4v_rmsnorm(const dsv4v_config* cfg, int64_t rows, const void* x, const float* w, void* y,
                           void* stream) {
  Shape s;
  DSV4V_TRY(check_config(cfg, s));
  if (rows < 0 || !x || !w || !y || !aligned16(x) || !aligned16(w) || !aligned16(y)) return DSV4V_ERR_INVALID_ARG;
  return cuda_status(
      launch_rmsnorm(s.bf16, x, w, y, rows, s.D, cfg->eps, static_cast<cudaStream_t>(stream)));
}

dsv4v_status dsv4v_qkv_rope(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* y, const void* wqkv,
                            const float* cos, const float* sin, void* qkv, void* workspace, size_t ws_bytes,
                            void* stream) {
  Ctx c;
  DSV4V_TRY(prepare(cfg, batch, workspace, ws_bytes, stream, c));
  if (!y || !wqkv || !cos || !sin || !qkv || !aligned16(y) || !aligned16(wqkv) || !aligned16(cos) ||
      !aligned16(sin) || !aligned16(qkv))
    return DSV4V_ERR_INVALID_ARG;
  const Shape& s = c.s;
  if (!s.bf16) {
    DSV4V_TRY(cuda_status(launch_gemm_f32(EPI_STORE, static_cast<const float*>(y), static_cast<const float*>(wqkv),
                                          nullptr, static_cast<float*>(qkv), nullptr, static_cast<int>(s.P), 3 * s.D,
                                          s.D, c.stream)));
    return cuda_status(launch_rope_apply_f32(static_cast<float*>(qkv), cos, sin, s.P, s.D, s.H, c.stream));
  }
  DSV4V_TRY(reset_counters(c));
  return gemm_bf16(c, EPI_QKV_ROPE, c.plans.qkv, y, s.P, s.D, wqkv, nullptr, 3 * s.D, qkv, nullptr, cos, sin);
}

dsv4v_status dsv4v_attention(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* qkv, void* out,
                             void* stream) {
  Ctx c;
  DSV4V_TRY(check_all(cfg, batch, c.s));
  if (!qkv || !out || !aligned16(qkv) || !aligned16(out)) return DSV4V_ERR_INVALID_ARG;
  if (!device_info(c.dev)) return DSV4V_ERR_CUDA;
  c.stream = static_cast<cudaStream_t>(stream);
  if (!c.s.bf16)
    return cuda_status(launch_attention_f32(static_cast<const float*>(qkv), static_cast<float*>(out),
                                            batch->cu_patches_dev, batch->n_images, c.s.P, c.s.D, c.s.H, c.stream));
  return attention_bf16(c, batch, qkv, out);
}

dsv4v_status dsv4v_linear_residual(const dsv4v_config* cfg, int64_t rows, int k, const void* a, const void* w,
                                   void* x, void* workspace, size_t ws_bytes, void* stream) {
  Ctx c;
  DSV4V_TRY(prepare_rows(cfg, rows, workspace, ws_bytes, stream, cfg && cfg->dtype == DSV4V_BF16, c));
  if (!a || !w || !x || !aligned16(a) || !aligned16(w) || !aligned16(x)) return DSV4V_ERR_INVALID_ARG;
  const Shape& s = c.s;
  if (k != s.D && k != s.F) return DSV4V_ERR_INVALID_ARG;
  if (!s.bf16)
    return cuda_status(launch_gemm_f32(EPI_RESID, static_cast<const float*>(a), static_cast<const float*>(w), nullptr,
                                       static_cast<float*>(x), static_cast<const float*>(x), static_cast<int>(rows),
                                       s.D, k, c.stream));
  DSV4V_TRY(reset_counters(c));
  const GemmPlan& plan = k == s.D ? c.plans.out : c.plans.down;
  return gemm_bf16(c, EPI_RESID, plan, a, rows, k, w, nullptr, s.D, x, x);
}

dsv4v_status dsv4v_swiglu(const dsv4v_config* cfg, int64_t rows, const void* y, const void* w_gate, const void* w_up,
                          void* h, void* workspace, size_t ws_bytes, void* stream) {
  Ctx c;
  DSV4V_TRY(prepare_rows(cfg, rows, workspace, ws_bytes, stream, cfg && cfg->dtype == DSV4V_BF16, c));
  if (!y || !w_gate || !w_up || !h || !aligned16(y) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(h))
    return DSV4V_ERR_INVALID_ARG;
  const Shape& s = c.s;
  if (!s.bf16)
    return cuda_status(launch_gemm_f32(EPI_SWIGLU, static_cast<const float*>(y), static_cast<const float*>(w_gate),
                                       static_cast<const float*>(w_up), static_cast<float*>(h), nullptr,
                                       static_cast<int>(rows), s.F, s.D, c.stream));
  DSV4V_TRY(reset_counters(c));
  return gemm_bf16(c, EPI_SWIGLU, c.plans.gateup, y, rows, s.D, w_gate, w_up, s.F, h, nullptr);
}

dsv4v_status dsv4v_patch_embed(const dsv4v_config* cfg, int64_t n_patches, int patch_h, int patch_w,
                               const void* patches, int64_t ld_patches, const void* w_proj, int64_t ld_w,
                               const float* bias, void* x_out, void* stream) {
  Ctx c;
  DSV4V_TRY(prepare_rows(cfg, n_patches, nullptr, 0, stream, false, c));
  if (patch_h <= 0 || patch_w <= 0 || patch_h > 64 || patch_w > 64) return DSV4V_ERR_INVALID_ARG;
  const int K = 3 * patch_h * patch_w;
  if (ld_patches == 0) ld_patches = K;
  if (ld_w == 0) ld_w = K;
  if (ld_patches < K || ld_w < K) return DSV4V_ERR_INVALID_ARG;
  if (n_patches == 0) return DSV4V_OK;
  if (!patches || !w_proj || !x_out || !aligned16(patches) || !aligned16(w_proj) || !aligned16(x_out) ||
      (bias && !aligned16(bias)))
    return DSV4V_ERR_INVALID_ARG;
  const Shape& s = c.s;
  if (!s.bf16) {
    if (ld_patches != K || ld_w != K) return DSV4V_ERR_UNSUPPORTED;
    return cuda_status(launch_gemm_f32(EPI_STORE, static_cast<const float*>(patches), static_cast<const float*>(w_proj),
                                       nullptr, static_cast<float*>(x_out), nullptr, static_cast<int>(n_patches), s.D,
                                       K, c.stream, bias));
  }
  // TMA rows start on 16-byte boundaries: strides in whole groups of 8 bf16.
  if (ld_patches % 8 || ld_w % 8) return DSV4V_ERR_UNSUPPORTED;
  // Whole tiles only (no split-tile scratch), so the call needs no workspace.
  const GemmPlan plan = plan_gemm(EPI_STORE, static_cast<int>(n_patches), s.D, K, c.dev.sms, 0);
  if (plan.bn == 0) return DSV4V_ERR_UNSUPPORTED;
  GemmExtra ex;
  ex.lda = ld_patches;
  ex.ldb = ld_w;
  ex.bias = bias;
  return gemm_bf16(c, EPI_STORE, plan, patches, n_patches, K, w_proj, nullptr, s.D, x_out, nullptr, nullptr, nullptr,
                   NormFold(), ex);
}

dsv4v_status dsv4v_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DSV4V_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v)) != cudaSuccess) return DSV4V_ERR_CUDA;
  if (v == 0) return DSV4V_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero)) != cudaSuccess) return DSV4V_ERR_CUDA;
  return v == kErrBridgeLayout ? DSV4V_ERR_LAYOUT : DSV4V_ERR_TIMEOUT;
}

// ---------------------------------------------------------------------------- image-token bridge
dsv4v_status dsv4v_image_layout(int grid_h, int grid_w, int downsample_ratio, int32_t* types_out, int64_t capacity,
                                int64_t* length_out) {
  if (grid_h < 1 || grid_w < 1 || downsample_ratio < 1) return DSV4V_ERR_INVALID_ARG;
  const int64_t rows = (grid_h + downsample_ratio - 1) / downsample_ratio;
  const int64_t cols = (grid_w + downsample_ratio - 1) / downsample_ratio;
  const int64_t len = 2 + rows * (cols + 1);
  if (length_out) *length_out = len;
  if (!types_out) return DSV4V_OK;
  if (capacity < len) return DSV4V_ERR_INVALID_ARG;
  int64_t q = 0;
  types_out[q++] = DSV4V_TOKEN_START;
  for (int64_t i = 0; i < rows; ++i) {
    for (int64_t j = 0; j < cols; ++j) types_out[q++] = DSV4V_TOKEN_IMAGE;
    types_out[q++] = DSV4V_TOKEN_NEWLINE;
  }
  types_out[q++] = DSV4V_TOKEN_END;
  return DSV4V_OK;
}

// Bridge scratch: per-chunk counts, then (visibility only) the span tables and the span number
// of every position.
struct BridgeLayout {
  size_t counts, span_first, span_last, span_of, total;
};

BridgeLayout bridge_layout(int64_t n) {
  BridgeLayout l{};
  const size_t chunks = static_cast<size_t>((n + kBridgeChunk - 1) / kBridgeChunk);
  const size_t ints = up256(static_cast<size_t>(n) * sizeof(int32_t));
  l.counts = 0;
  l.span_first = up256(chunks * sizeof(int4));
  l.span_last = l.span_first + ints;
  l.span_of = l.span_last + ints;
  l.total = l.span_of + ints;
  return l;
}

size_t dsv4v_bridge_workspace_size(int64_t n_positions) {
  if (n_positions < 1 || n_positions >= (int64_t{1} << 31)) return 0;
  return bridge_layout(n_positions).total;
}

dsv4v_status dsv4v_merge_image_embeddings(const dsv4v_config* cfg, const dsv4v_batch* batch, int64_t n_seqs,
                                          int64_t seq_len, const int32_t* token_types, const void* image_tokens,
                                          const void* sentinels, void* embeds, void* workspace, size_t ws_bytes,
                                          void* stream) {
  Shape s;
  DSV4V_TRY(check_all(cfg, batch, s));
  if (n_seqs < 1 || seq_len < 1 || n_seqs > (int64_t{1} << 31) / seq_len) return DSV4V_ERR_INVALID_ARG;
  const int64_t n = n_seqs * seq_len;
  if (n >= (int64_t{1} << 31)) return DSV4V_ERR_INVALID_ARG;
  if (!token_types || (reinterpret_cast<uintptr_t>(token_types) & 3u)) return DSV4V_ERR_INVALID_ARG;
  for (const void* ptr : {image_tokens, sentinels, static_cast<const void*>(embeds)})
    if (!ptr || !aligned16(ptr)) return DSV4V_ERR_INVALID_ARG;
  const size_t row_bytes = static_cast<size_t>(s.E) * (s.bf16 ? 2 : 4);
  if (row_bytes % 16) return DSV4V_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < dsv4v_bridge_workspace_size(n))
    return DSV4V_ERR_WORKSPACE;
  DeviceInfo d;
  if (!device_info(d)) return DSV4V_ERR_CUDA;
  return cuda_status(launch_bridge_merge(token_types, n, seq_len, static_cast<int4*>(workspace), batch->grid_hw_dev,
                                         batch->n_images, s.r, s.T, image_tokens, sentinels, embeds,
                                         static_cast<int>(row_bytes / 16), d.err, static_cast<cudaStream_t>(stream)));
}

dsv4v_status dsv4v_image_visibility(int64_t n_seqs, int64_t seq_len, const int32_t* token_types, void* mask,
                                    int elem_bytes, void* workspace, size_t ws_bytes, void* stream) {
  if (n_seqs < 1 || seq_len < 1 || n_seqs > (int64_t{1} << 31) / seq_len) return DSV4V_ERR_INVALID_ARG;
  const int64_t n = n_seqs * seq_len;
  if (n >= (int64_t{1} << 31)) return DSV4V_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return DSV4V_ERR_INVALID_ARG;
  if (!token_types || (reinterpret_cast<uintptr_t>(token_types) & 3u)) return DSV4V_ERR_INVALID_ARG;
  if (!mask || (reinterpret_cast<uintptr_t>(mask) & static_cast<uintptr_t>(elem_bytes - 1)))
    return DSV4V_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < dsv4v_bridge_workspace_size(n))
    return DSV4V_ERR_WORKSPACE;
  DeviceInfo d;
  if (!device_info(d)) return DSV4V_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const BridgeLayout l = bridge_layout(n);
  return cuda_status(launch_image_visibility(
      token_types, n_seqs, seq_len, mask, elem_bytes, reinterpret_cast<int4*>(ws + l.counts),
      reinterpret_cast<int32_t*>(ws + l.span_first), reinterpret_cast<int32_t*>(ws + l.span_last),
      reinterpret_cast<int32_t*>(ws + l.span_of), d.err, static_cast<cudaStream_t>(stream)));
}

dsv4v_status dsv4v_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  DeviceInfo d;
  if (!device_info(d)) return DSV4V_ERR_CUDA;
  if (limit_ns > 10000000000ull) return DSV4V_ERR_INVALID_ARG;
  return cuda_status(launch_selftest_wait(limit_ns, d.err, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------- backward
namespace {

constexpr int kNormParts = 512;  // most CTAs of one RMSNorm backward (each leaves a [D] partial)

// Scratch of the backward calls, after the forward layout (whose split-tile scratch and
// rotation tables the recompute reuses).  Activations and gradients are bf16 [P, width]; fp32
// attention row statistics and RMSNorm partials.  The gradient GEMMs read every operand where
// it lies (MN-major where needed), so there are no transposed copies.
struct BwdLayout {
  size_t y1, qkv, att, x2, y2, g, u, h, dh, dgu, dy2, dx2, datt, dqkv, dy1, dcur0, dcur1;
  size_t lse, rowdot, norm_parts, total;
};

BwdLayout bwd_layout(const Shape& s, size_t fwd_total) {
  BwdLayout l{};
  const size_t P = static_cast<size_t>(s.P), D = s.D, F = s.F;
  size_t off = up256(fwd_total);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += up256(bytes);
    return at;
  };
  l.y1 = take(P * D * 2);
  l.qkv = take(P * 3 * D * 2);
  l.att = take(P * D * 2);
  l.x2 = take(P * D * 2);
  l.y2 = take(P * D * 2);
  l.g = take(P * F * 2);
  l.u = take(P * F * 2);
  l.h = take(P * F * 2);
  l.dh = take(P * F * 2);
  l.dgu = take(P * 2 * F * 2);
  l.dy2 = take(P * D * 2);
  l.dx2 = take(P * D * 2);
  l.datt = take(P * D * 2);
  l.dqkv = take(P * 3 * D * 2);
  l.dy1 = take(P * D * 2);
  l.dcur0 = take(P * D * 2);
  l.dcur1 = take(P * D * 2);
  l.lse = take(P * s.H * 4);
  l.rowdot = take(P * s.H * 4);
  l.norm_parts = take(static_cast<size_t>(kNormParts) * D * 4);
  l.total = off;
  return l;
}

// The backward calls are bf16 only.
dsv4v_status bwd_prepare(const dsv4v_config* cfg, const dsv4v_batch* batch, void* workspace, size_t ws_bytes,
                         void* stream, Ctx& c, BwdLayout& bl) {
  DSV4V_TRY(check_all(cfg, batch, c.s));
  if (!c.s.bf16) return DSV4V_ERR_UNSUPPORTED;
  DSV4V_TRY(prepare(cfg, batch, workspace, ws_bytes, stream, c));
  bl = bwd_layout(c.s, c.lay.total);
  if (ws_bytes < bl.total) return DSV4V_ERR_WORKSPACE;
  return DSV4V_OK;
}

int norm_parts_for(const Ctx& c, int64_t rows) {
  const int64_t want = std::min<int64_t>((rows + 7) / 8, 2 * static_cast<int64_t>(c.dev.sms));
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, kNormParts)));
}

// out[M, n_out] = a[M, K] . b[n_out, K]^T with row strides lda / ldb (0 = K): whole tiles only,
// so no split-tile scratch is used.
dsv4v_status gemm_store(const Ctx& c, const void* a, int64_t M, int K, int64_t lda, const void* b, int64_t ldb,
                        int n_out, void* out) {
  const GemmPlan plan = plan_gemm(EPI_STORE, static_cast<int>(M), n_out, K, c.dev.sms, 0);
  if (plan.bn == 0) return DSV4V_ERR_UNSUPPORTED;
  GemmExtra ex;
  ex.lda = lda;
  ex.ldb = ldb;
  ex.b_early = false;  // B is an activation or a transposed copy written earlier in the call
  return gemm_bf16(c, EPI_STORE, plan, a, M, K, b, nullptr, n_out, out, nullptr, nullptr, nullptr, NormFold(), ex);
}

// out[M, n_out] = A . B with either operand given as its stored matrix (MN-major, no transposed
// copy): a_mn, A is stored [K, M] (row stride lda), else [M, K]; b_mn, B is stored [K, n_out]
// (row stride ldb; with b2, its rows from kb_split * 64 on are b2's rows), else [n_out, K].
dsv4v_status gemm_store_mn(const Ctx& c, const void* a, int64_t M, int K, int64_t lda, bool a_mn, const void* b,
                           int64_t ldb, bool b_mn, int n_out, void* out, const void* b2 = nullptr, int kb_split = 0) {
  // With A K-major (input gradients, whose K can be long) the planner's cluster split-K plans
  // are allowed too; with an MN-major A (weight gradients, K = the packed rows) whole tiles.
  GemmPlan plan{};
  if (!a_mn) plan = plan_gemm(EPI_STORE, static_cast<int>(M), n_out, K, c.dev.sms, 0);
  if (a_mn || plan.bn == 192 || plan.bn == 0 || (plan.ks > 1 && !b_mn))
    plan = plan_gemm_whole(static_cast<int>(M), n_out, K, c.dev.sms);
  if (plan.bn == 0) return DSV4V_ERR_UNSUPPORTED;
  GemmExtra ex;
  ex.lda = lda;
  ex.ldb = ldb;
  ex.b_early = false;  // B may be an activation written earlier in the call
  ex.a_mn = a_mn;
  ex.b_mn = b_mn;
  ex.kb_split = kb_split;
  return gemm_bf16(c, EPI_STORE, plan, a, M, K, b, b2, n_out, out, nullptr, nullptr, nullptr, NormFold(), ex);
}



// Attention backward on tcgen05.  lse_ready: bl.lse already holds the forward's per-row
// log-sum-exp ([H, P], written by the forward recompute); otherwise the forward runs once more
// into scratch to produce it.
dsv4v_status attention_bwd(const Ctx& c, const BwdLayout& bl, const dsv4v_batch* b, const void* qkv, const void* out,
                           const void* dout, void* dqkv, bool lse_ready) {
  if (!lse_ready) DSV4V_TRY(attention_bf16(c, b, qkv, c.at<void>(c.lay.attn), c.at<float>(bl.lse)));
  CUtensorMap tm_qkv, tm_do;
  if (!bf16_map(qkv, c.s.P, 3 * c.s.D, 128, &tm_qkv) || !bf16_map(dout, c.s.P, c.s.D, 128, &tm_do))
    return DSV4V_ERR_CUDA;
  thread_local AttnSchedule sched;
  attention_schedule(b, 1, 1, sched);
  return cuda_status(launch_attention_bwd_tc(&tm_qkv, &tm_do, sched, sched, out, dout, c.at<float>(bl.lse),
                                             c.at<float>(bl.rowdot), c.s.P, dqkv, c.s.P, c.s.H, c.s.D, c.dev.err,
                                             c.stream));
}

dsv4v_status rmsnorm_bwd(const Ctx& c, const BwdLayout& bl, const void* x, const float* w, const void* dy,
                         const void* d_in, void* dx, float* dw) {
  return cuda_status(launch_rmsnorm_bwd(x, w, dy, d_in, dx, c.at<float>(bl.norm_parts), norm_parts_for(c, c.s.P), dw,
                                        c.s.P, c.s.D, c.eps, c.stream));
}

bool grads_ok(const dsv4v_block_grads* g) {
  if (!g) return false;
  const void* ptrs[] = {g->norm1_w, g->wqkv, g->wo, g->norm2_w, g->w_gate, g->w_up, g->w_down};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return false;
  return true;
}

// One block backward (see dsv4v_block_backward): recompute, then the MLP branch, norm2, the
// output projection, attention, the rotation and projection, norm1.
dsv4v_status block_backward_bf16(const Ctx& c, const BwdLayout& bl, const dsv4v_batch* batch,
                                 const dsv4v_block_weights* w, const float* cos, const float* sin, const void* x,
                                 const void* dout, void* dx, const dsv4v_block_grads* gr) {
  const Shape& s = c.s;
  const int64_t P = s.P;
  const int D = s.D, F = s.F;
  void* y1 = c.at<void>(bl.y1);
  void* qkv = c.at<void>(bl.qkv);
  void* att = c.at<void>(bl.att);
  void* x2 = c.at<void>(bl.x2);
  void* y2 = c.at<void>(bl.y2);
  void* g = c.at<void>(bl.g);
  void* u = c.at<void>(bl.u);
  void* h = c.at<void>(bl.h);
  void* dh = c.at<void>(bl.dh);
  uint8_t* dgu = c.at<uint8_t>(bl.dgu);
  void* dy2 = c.at<void>(bl.dy2);
  void* dx2 = c.at<void>(bl.dx2);
  void* datt = c.at<void>(bl.datt);
  void* dqkv = c.at<void>(bl.dqkv);
  void* dy1 = c.at<void>(bl.dy1);
  const int Pk = static_cast<int>(P);  // K of the weight-gradient GEMMs (they reduce over the rows)
  // recompute the block's intermediates
  DSV4V_TRY(cuda_status(launch_rmsnorm(true, x, w->norm1_w, y1, P, D, c.eps, c.stream)));
  DSV4V_TRY(reset_counters(c));
  DSV4V_TRY(gemm_bf16(c, EPI_QKV_ROPE, c.plans.qkv, y1, P, D, w->wqkv, nullptr, 3 * D, qkv, nullptr, cos, sin));
  DSV4V_TRY(attention_bf16(c, batch, qkv, att, c.at<float>(bl.lse)));
  DSV4V_TRY(cuda_status(cudaMemcpyAsync(x2, x, static_cast<size_t>(P) * D * 2, cudaMemcpyDeviceToDevice, c.stream)));
  DSV4V_TRY(reset_counters(c));
  DSV4V_TRY(gemm_bf16(c, EPI_RESID, c.plans.out, att, P, D, w->wo, nullptr, D, x2, x2));
  DSV4V_TRY(cuda_status(launch_rmsnorm(true, x2, w->norm2_w, y2, P, D, c.eps, c.stream)));
  DSV4V_TRY(gemm_store(c, y2, P, D, 0, w->w_gate, 0, F, g));
  DSV4V_TRY(gemm_store(c, y2, P, D, 0, w->w_up, 0, F, u));
  // MLP branch.  Input gradients read each weight as stored ([K, n]: MN-major B); weight
  // gradients reduce over the rows and read both the output gradient and the activation as
  // stored ([P, width]: MN-major A and B), so no operand is transposed.
  DSV4V_TRY(gemm_store_mn(c, dout, P, D, 0, false, w->w_down, F, true, F, dh));  // dh = dout . w_down
  DSV4V_TRY(cuda_status(launch_swiglu_bwd(g, u, dh, dgu, h, P, F, c.dev.sms, c.stream)));
  DSV4V_TRY(gemm_store_mn(c, dout, D, Pk, D, true, h, F, true, F, gr->w_down));  // dout^T . h
  // dy2 = [dg | du] . [w_gate; w_up]: B's K rows continue from w_gate into w_up (F % 64 == 0)
  DSV4V_TRY(gemm_store_mn(c, dgu, P, 2 * F, 0, false, w->w_gate, D, true, D, dy2, w->w_up, F / 64));
  DSV4V_TRY(gemm_store_mn(c, dgu, F, Pk, 2 * F, true, y2, D, true, D, gr->w_gate));  // dg^T . y2
  DSV4V_TRY(gemm_store_mn(c, dgu + static_cast<size_t>(F) * 2, F, Pk, 2 * F, true, y2, D, true, D,
                          gr->w_up));  // du^T . y2
  // norm2 and the residual
  DSV4V_TRY(rmsnorm_bwd(c, bl, x2, w->norm2_w, dy2, dout, dx2, gr->norm2_w));
  // output projection
  DSV4V_TRY(gemm_store_mn(c, dx2, P, D, 0, false, w->wo, D, true, D, datt));      // dx2 . wo
  DSV4V_TRY(gemm_store_mn(c, dx2, D, Pk, D, true, att, D, true, D, gr->wo));      // dx2^T . att
  // attention, rotation, fused projection
  DSV4V_TRY(attention_bwd(c, bl, batch, qkv, att, datt, dqkv, true));
  DSV4V_TRY(cuda_status(launch_rotary_bwd(dqkv, cos, sin, P, D, s.hd, c.dev.sms, c.stream)));
  DSV4V_TRY(gemm_store_mn(c, dqkv, P, 3 * D, 0, false, w->wqkv, D, true, D, dy1));     // dqkv . wqkv
  DSV4V_TRY(gemm_store_mn(c, dqkv, 3 * D, Pk, 3 * D, true, y1, D, true, D, gr->wqkv));  // dqkv^T . y1
  // norm1 and the residual
  return rmsnorm_bwd(c, bl, x, w->norm1_w, dy1, dx2, dx, gr->norm1_w);
}

}  // namespace

size_t dsv4v_backward_workspace_size(const dsv4v_config* cfg, const dsv4v_batch* batch) {
  Shape s;
  if (check_all(cfg, batch, s) != DSV4V_OK || !s.bf16) return 0;
  DeviceInfo d;
  const int sms = device_info(d) ? d.sms : planning_sms();
  return bwd_layout(s, make_layout(s, make_plans(s, sms)).total).total;
}

dsv4v_status dsv4v_attention_backward(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* qkv,
                                      const void* out, const void* d_out, void* dqkv, void* workspace, size_t ws_bytes,
                                      void* stream) {
  Ctx c;
  BwdLayout bl;
  DSV4V_TRY(bwd_prepare(cfg, batch, workspace, ws_bytes, stream, c, bl));
  for (const void* p : {qkv, out, d_out, static_cast<const void*>(dqkv)})
    if (!p || !aligned16(p)) return DSV4V_ERR_INVALID_ARG;
  return attention_bwd(c, bl, batch, qkv, out, d_out, dqkv, false);
}

dsv4v_status dsv4v_rmsnorm_backward(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* x, const float* w,
                                    const void* dy, const void* d_in, void* dx, float* dw, void* workspace,
                                    size_t ws_bytes, void* stream) {
  Ctx c;
  BwdLayout bl;
  DSV4V_TRY(bwd_prepare(cfg, batch, workspace, ws_bytes, stream, c, bl));
  for (const void* p : {x, static_cast<const void*>(w), dy, static_cast<const void*>(dx), static_cast<const void*>(dw)})
    if (!p || !aligned16(p)) return DSV4V_ERR_INVALID_ARG;
  if (d_in && !aligned16(d_in)) return DSV4V_ERR_INVALID_ARG;
  return rmsnorm_bwd(c, bl, x, w, dy, d_in, dx, dw);
}

dsv4v_status dsv4v_block_backward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                  const dsv4v_block_weights* weights, const float* cos, const float* sin, const void* x,
                                  const void* d_out, void* dx, const dsv4v_block_grads* grads, void* workspace,
                                  size_t ws_bytes, void* stream) {
  Ctx c;
  BwdLayout bl;
  DSV4V_TRY(bwd_prepare(cfg, batch, workspace, ws_bytes, stream, c, bl));
  if (!weights_ok(weights) || !grads_ok(grads) || !cos || !sin || !aligned16(cos) || !aligned16(sin))
    return DSV4V_ERR_INVALID_ARG;
  for (const void* p : {x, d_out, static_cast<const void*>(dx)})
    if (!p || !aligned16(p)) return DSV4V_ERR_INVALID_ARG;
  return block_backward_bf16(c, bl, batch, weights, cos, sin, x, d_out, dx, grads);
}

dsv4v_status dsv4v_tower_backward(const dsv4v_config* cfg, const dsv4v_batch* batch, const dsv4v_block_weights* layers,
                                  const float* final_norm_w, const void* const* layer_inputs, const void* x_last,
                                  const void* d_out, void* dx, const dsv4v_block_grads* layer_grads,
                                  float* d_final_norm_w, void* workspace, size_t ws_bytes, void* stream) {
  Ctx c;
  BwdLayout bl;
  DSV4V_TRY(bwd_prepare(cfg, batch, workspace, ws_bytes, stream, c, bl));
  const int L = c.s.L;
  if (L < 1 || !layers || !layer_inputs || !layer_grads || !d_out || !dx || !aligned16(d_out) || !aligned16(dx))
    return DSV4V_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (!weights_ok(&layers[l]) || !grads_ok(&layer_grads[l]) || !layer_inputs[l] || !aligned16(layer_inputs[l]))
      return DSV4V_ERR_INVALID_ARG;
  if (final_norm_w && (!aligned16(final_norm_w) || !x_last || !aligned16(x_last) || !d_final_norm_w ||
                       !aligned16(d_final_norm_w)))
    return DSV4V_ERR_INVALID_ARG;
  float* cos = c.at<float>(c.lay.cos);
  float* sin = c.at<float>(c.lay.sin);
  DSV4V_TRY(rope_table(c, batch, cos, sin));
  const void* d = d_out;
  void* bufs[2] = {c.at<void>(bl.dcur0), c.at<void>(bl.dcur1)};
  int next = 0;
  if (final_norm_w) {
    DSV4V_TRY(rmsnorm_bwd(c, bl, x_last, final_norm_w, d_out, nullptr, bufs[next], d_final_norm_w));
    d = bufs[next];
    next ^= 1;
  }
  for (int l = L - 1; l >= 0; --l) {
    void* target = l == 0 ? dx : bufs[next];
    DSV4V_TRY(block_backward_bf16(c, bl, batch, &layers[l], cos, sin, layer_inputs[l], d, target, &layer_grads[l]));
    d = target;
    next ^= 1;
  }
  return DSV4V_OK;
}

}  // extern "C"
