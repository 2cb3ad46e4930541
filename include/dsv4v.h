/*
 * dsv4v -- C ABI of a B200 (sm_100a) forward pass of the DeepSeek-V4-Flash vision tower
 * and aligner.
 *
 * Sources (page title, then section):
 *   [vision-API]  "nemo_automodel.components.models.deepseek_v4.vision" API reference
 *   [model-API]   "nemo_automodel.components.models.deepseek_v4.model" API reference
 *   [PR]          NeMo-Automodel pull request adding DeepSeek-V4-Flash-Vision-Exp
 *                 (Changelog, Validation)
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Packed varlen layout.  The patches of all images of a batch are stored back to back:
 *    activations are row-major [P, vision_dim] with P = sum_i n_h[i] * n_w[i].  Inside an image
 *    patch p = h * n_w + w (row-major over the grid, as the [n_h * n_w, vision_dim] layouts of
 *    [vision-API, DeepseekV4VisionTransformer.forward] imply).  Offsets follow the cu_seqlens
 *    form of [model-API, THD packing helpers]: int32, n_images + 1 entries, cu[0] = 0,
 *    cu[i + 1] - cu[i] = n_h[i] * n_w[i].
 *  - Images never interact: attention and the aligner merge stay inside an image, so packing
 *    several images changes no result.
 *  - Weights are row-major [out_features, in_features] (nn.Linear layout).  wqkv stacks the q,
 *    k and v projections as three blocks of vision_dim rows, head-major inside each block.
 *    RMSNorm scales are always fp32.  Every projection is bias-free.
 *  - dtype DSV4V_BF16: activations, residual stream and projection weights are bf16; GEMMs
 *    accumulate in fp32; RMSNorm, the rotary rotation, softmax and SiLU run in fp32 and round
 *    once to bf16.  dtype DSV4V_F32: everything fp32 (CUDA-core path for small widths).
 *  - The caller owns every buffer.  All device pointers must be on the current CUDA device.
 *    The library allocates no device memory; scratch space is the caller's `workspace`
 *    (size from dsv4v_workspace_size, 256-byte aligned).
 *  - Every call is asynchronous and ordered on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Argument, shape and workspace errors are reported synchronously, before any
 *    kernel is launched.  A device-side check that fails (a bounded wait that gives up)
 *    records an error that dsv4v_device_error() returns after synchronising the stream.
 *  - Calls on the same workspace must not overlap on the GPU (put them on one stream).
 *  - This library's kernels may start while earlier ones of the library on the stream still
 *    run (dependent launch), and may read their weight arguments before those finish;
 *    everything else they read only after.  So a weight passed to a call must not have been
 *    written by this library's kernels since the last other kernel (or host synchronisation)
 *    on the stream; an optimizer step in between is enough.
 *  - No call keeps device state between calls; each call may be captured in a CUDA graph
 *    (the launch geometry is taken from the host copies of the grids and offsets, which must
 *    equal the device copies).
 */
#ifndef DSV4V_H
#define DSV4V_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSV4V_OK = 0,
  DSV4V_ERR_INVALID_ARG = 1,   /* null pointer, bad grid/offset, inconsistent sizes */
  DSV4V_ERR_UNSUPPORTED = 2,   /* shape outside the constraints listed at the config below */
  DSV4V_ERR_WORKSPACE = 3,     /* workspace NULL, misaligned or smaller than required */
  DSV4V_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  DSV4V_ERR_TIMEOUT = 5,       /* a device-side check failed: a bounded wait gave up, or the two
                                  CTAs of a GEMM CTA pair got different TMEM addresses (see
                                  dsv4v_device_error) */
  DSV4V_ERR_LAYOUT = 6         /* pseudo-token types that do not fit the images, found on the
                                  device by dsv4v_merge_image_embeddings or
                                  dsv4v_image_visibility (see dsv4v_device_error) */
} dsv4v_status;

typedef enum { DSV4V_F32 = 0, DSV4V_BF16 = 1 } dsv4v_dtype;

/* Model dimensions ([vision-API] DeepseekV4VisionAttention: head_dim = vision_dim / n_heads;
 * DeepseekV4VisionAligner: downsample_ratio; DeepseekV4VisionRMSNorm: eps default 1e-6;
 * DeepseekV4VisionTransformer: rope_theta).
 * Constraints: all sizes > 0; vision_dim % n_heads == 0; head_dim % 4 == 0 (the 2D table
 * splits head_dim / 2 angles between rows and columns).
 * DSV4V_BF16 additionally: head_dim == 64, vision_dim % 128 == 0, mlp_hidden % 128 == 0,
 * llm_dim % 128 == 0.  Otherwise DSV4V_ERR_UNSUPPORTED. */
typedef struct {
  int vision_dim;        /* D */
  int n_heads;           /* H */
  int mlp_hidden;        /* F, SwiGLU hidden width */
  int downsample_ratio;  /* r, aligner merges r x r patches */
  int llm_dim;           /* E, aligner output width */
  int n_layers;          /* L, blocks in the tower */
  float eps;             /* RMSNorm epsilon (1e-6) */
  float rope_theta;      /* rotary base (10000) */
  dsv4v_dtype dtype;
} dsv4v_config;

/* One block's parameters ([vision-API] DeepseekV4VisionBlock: norm1, attn.wqkv, output
 * projection, norm2, mlp).  Scales are fp32 [D]; projections are in the config dtype:
 * wqkv [3D, D], wo [D, D], w_gate [F, D], w_up [F, D], w_down [D, F].  Device pointers, each
 * 16-byte aligned. */
typedef struct {
  const float* norm1_w;
  const float* norm2_w;
  const void* wqkv;
  const void* wo;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
} dsv4v_block_weights;

/* A packed batch of images.  grid_hw: [n_images, 2] int32 (n_h, n_w), each >= 1.  cu_patches:
 * [n_images + 1] int32 offsets (see above).  Both are needed on the host (launch geometry and
 * validation) and on the device (read by the kernels); the two copies must hold the same
 * values.  1 <= n_images <= DSV4V_MAX_IMAGES. */
typedef struct {
  int n_images;
  const int32_t* grid_hw_host;
  const int32_t* grid_hw_dev;
  const int32_t* cu_patches_host;
  const int32_t* cu_patches_dev;
} dsv4v_batch;

#define DSV4V_MAX_IMAGES 1024

/* Bytes of device scratch that every call below needs for this config and batch (the maximum
 * over the calls, so one workspace serves all of them).  0 if the arguments are invalid. */
size_t dsv4v_workspace_size(const dsv4v_config* cfg, const dsv4v_batch* batch);

/* [vision-API, get_vision_cos_sin]: the 2D rotary table of every image of the batch, stacked
 * in packing order: row p holds the table row of packed patch p.  Reading adopted: the table
 * width is head_dim / 2; the first head_dim / 4 angles are h * theta^(-k / (head_dim/4)) and
 * the last head_dim / 4 are w * theta^(-k / (head_dim/4)), k < head_dim / 4, with (h, w) the
 * patch's grid position inside its own image.
 * cos_out, sin_out: device fp32 [P, head_dim / 2], written. */
dsv4v_status dsv4v_rope2d_table(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                float* cos_out, float* sin_out, void* stream);

/* [vision-API, DeepseekV4VisionBlock.forward]: one pre-norm block on the packed batch,
 *   x <- x + wo . attn(rope(wqkv . norm1(x)))   (attention within each image only)
 *   x <- x + w_down . (silu(w_gate . norm2(x)) * (w_up . norm2(x)))
 * cos, sin: device fp32 [P, head_dim / 2] (dsv4v_rope2d_table).  x_inout: device [P, D] in the
 * config dtype, updated in place.  workspace: device scratch of ws_bytes bytes. */
dsv4v_status dsv4v_block_forward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                 const dsv4v_block_weights* weights, const float* cos,
                                 const float* sin, void* x_inout, void* workspace,
                                 size_t ws_bytes, void* stream);

/* [vision-API, DeepseekV4VisionTransformer.forward] from patch states on: builds the rotary
 * table, runs cfg->n_layers blocks (layers: host array of n_layers weight structs), then the
 * tower's final RMSNorm with final_norm_w (device fp32 [D]; NULL skips it).  x_inout: device
 * [P, D], updated in place.  The patch embedding is not part of this call. */
dsv4v_status dsv4v_tower_forward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                 const dsv4v_block_weights* layers, const float* final_norm_w,
                                 void* x_inout, void* workspace, size_t ws_bytes, void* stream);

/* [vision-API, DeepseekV4VisionAligner.forward]: per image, zero-pad the grid at the
 * bottom/right to a multiple of r (a stated assumption for odd grids), merge each r x r window
 * into one token whose channel (a * r + b) * D + c holds channel c of the patch at window
 * position (a, b) (a = row offset), order tokens row-major, and project with
 * w_align [E, r*r*D] (bias-free).
 * x: device [P, D]; out: device [T, E] with T = sum_i ceil(n_h/r) * ceil(n_w/r), both in the
 * config dtype.  cu_tokens_host: optional host int32 [n_images + 1], filled with the token
 * offsets of each image (NULL to skip). */
dsv4v_status dsv4v_aligner_forward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                   const void* x, const void* w_align, void* out,
                                   int32_t* cu_tokens_host, void* workspace, size_t ws_bytes,
                                   void* stream);

/* Number of aligner tokens T of the batch (host computation); -1 if the arguments are
 * invalid. */
int64_t dsv4v_aligner_tokens(const dsv4v_config* cfg, const dsv4v_batch* batch);

/* Kernel classes that dsv4v_tower_forward_profiled brackets with events. */
enum {
  DSV4V_PROFILE_QKV = 0,        /* fused projection + rotation GEMM (norm1 folded in) */
  DSV4V_PROFILE_ATTENTION = 1,  /* varlen attention */
  DSV4V_PROFILE_OUT = 2,        /* output projection + residual (prepares norm2) */
  DSV4V_PROFILE_SWIGLU = 3,     /* gate/up GEMM + silu*mul (norm2 folded in) */
  DSV4V_PROFILE_DOWN = 4,       /* down projection + residual (prepares the next norm1) */
  DSV4V_PROFILE_CHAIN = 5,      /* chained GEMMs of one block in one persistent launch (output
                                   projection, SwiGLU, down projection and the next block's
                                   q|k|v projection); see dsv4v_tower_path */
  DSV4V_PROFILE_KINDS = 6
};

/* Number of kernel launches that dsv4v_tower_forward (with a final norm when final_norm != 0)
 * followed by dsv4v_aligner_forward (when aligner != 0) put on the stream for this config and
 * batch under the current launch-sequence setting (host computation); -1 if the arguments are
 * invalid. */
int dsv4v_step_launches(const dsv4v_config* cfg, const dsv4v_batch* batch, int final_norm, int aligner);

/* Launch sequence of the bf16 blocks (no effect on fp32 configs).  Both compute the same
 * block, with the same roundings: they differ in how the GEMMs' K dimension is split, so sums
 * of fp32 products may be added in another order.
 *  DSV4V_PATH_KERNELS: one kernel per GEMM of the block (plus attention).
 *  DSV4V_PATH_CHAIN:   per block, attention plus one persistent launch that runs the output
 *                      projection, SwiGLU, the down projection and the next block's q|k|v
 *                      projection with per-128-row-tile dependencies between them.
 *  DSV4V_PATH_AUTO:    the sequence measured faster for the batch's size (at present one kernel
 *                      per GEMM at every size). */
enum { DSV4V_PATH_AUTO = 0, DSV4V_PATH_KERNELS = 1, DSV4V_PATH_CHAIN = 2 };

/* Sets the launch sequence for the calls that follow, process-wide (host state only; the
 * default is DSV4V_PATH_AUTO).  Workspace sizes depend on it: size the workspace after setting
 * it.  Returns DSV4V_ERR_INVALID_ARG for an unknown value. */
dsv4v_status dsv4v_set_tower_path(int path);

/* Graph replay of the step calls (dsv4v_tower_forward, dsv4v_aligner_forward).  Each host
 * thread keeps up to 16 CUDA graph executables keyed by every argument that shapes a call's launches:
 * the config and batch values, the batch's device pointers, the weight, buffer and workspace
 * pointers, the launch sequence (dsv4v_set_tower_path) and the current device.  The first call
 * with a key launches its kernels directly; the second captures them on the caller's stream
 * (thread-local capture mode) and launches the graph; later calls launch the graph.  The data
 * behind the pointers may change freely between calls; the graph reads it when it runs.  Calls
 * on the legacy default stream (NULL), on cudaStreamPerThread, or on a stream that is being
 * captured (the caller's own graph) always launch directly.  A capture or instantiation that
 * fails leaves that key on direct launches (the call still runs).
 * dsv4v_set_graph_replay(0) turns the cache off for the calls that follow (process-wide host
 * state; default on); dsv4v_release_graphs() destroys the calling thread's cached executables
 * (one still running is freed when it completes); a thread that exits without calling it leaves
 * its executables to the driver's teardown.  Neither needs a GPU or fails. */
void dsv4v_set_graph_replay(int enable);
void dsv4v_release_graphs(void);

/* The launch sequence dsv4v_block_forward / dsv4v_tower_forward use for this config and
 * batch under the current setting: DSV4V_PATH_KERNELS or DSV4V_PATH_CHAIN; -1 if the arguments
 * are invalid. */
int dsv4v_tower_path(const dsv4v_config* cfg, const dsv4v_batch* batch);

/* dsv4v_tower_forward, recording CUDA events around the launches of every layer:
 * events[(layer * DSV4V_PROFILE_KINDS + kind) * 2 + 0] before and [... + 1] after the kernel
 * of that class (cudaEvent_t handles passed as void*, created by the caller; NULL entries are
 * skipped).  With DSV4V_PATH_KERNELS the kinds QKV, ATTENTION, OUT, SWIGLU and DOWN are
 * recorded; with DSV4V_PATH_CHAIN, ATTENTION and CHAIN (layer l's CHAIN launch runs its output
 * projection, SwiGLU and down projection and layer l + 1's q|k|v projection; layer 0's q|k|v
 * projection is a launch of its own that is not bracketed).  The events sit between kernels, so the bracketed kernels cannot overlap their
 * neighbours as in dsv4v_tower_forward; per-kernel durations from them are standalone
 * durations.  Same results as dsv4v_tower_forward. */
dsv4v_status dsv4v_tower_forward_profiled(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                          const dsv4v_block_weights* layers, const float* final_norm_w,
                                          void* x_inout, void* workspace, size_t ws_bytes, void* stream,
                                          void* const* events);

/* ---- Component entry points: single steps of the block, for testing and profiling. ---- */

/* RMSNorm [vision-API, DeepseekV4VisionRMSNorm]: y = w * x / sqrt(mean(x^2) + eps) per row,
 * computed in fp32, cast to the config dtype.  x, y: device [rows, D]; w: device fp32 [D].
 * y may equal x. */
dsv4v_status dsv4v_rmsnorm(const dsv4v_config* cfg, int64_t rows, const void* x,
                           const float* w, void* y, void* stream);

/* Fused projection + rotation ([vision-API, DeepseekV4VisionAttention.wqkv] and
 * apply_vision_rotary): qkv = y . wqkv^T, then q and k (columns [0, 2D)) rotated with the
 * half-split rule x'_j = x_j cos_j - x_{j+hd/2} sin_j, x'_{j+hd/2} = x_{j+hd/2} cos_j +
 * x_j sin_j.  y: device [P, D]; qkv: device [P, 3D], config dtype. */
dsv4v_status dsv4v_qkv_rope(const dsv4v_config* cfg, const dsv4v_batch* batch, const void* y,
                            const void* wqkv, const float* cos, const float* sin, void* qkv,
                            void* workspace, size_t ws_bytes, void* stream);

/* Full bidirectional attention within each image ([vision-API, DeepseekV4VisionAttention]):
 * out[:, h*hd:(h+1)*hd] = softmax(q_h k_h^T / sqrt(hd)) v_h per image and head.
 * qkv: device [P, 3D] (q | k | v, already rotated); out: device [P, D]. */
dsv4v_status dsv4v_attention(const dsv4v_config* cfg, const dsv4v_batch* batch,
                             const void* qkv, void* out, void* stream);

/* Projection with residual add: x <- x + a . w^T.  a: device [rows, K]; w: device [D, K];
 * x: device [rows, D].  K is vision_dim or mlp_hidden. */
dsv4v_status dsv4v_linear_residual(const dsv4v_config* cfg, int64_t rows, int k,
                                   const void* a, const void* w, void* x, void* workspace,
                                   size_t ws_bytes, void* stream);

/* PatchMerger projector (the second aligner the pages describe: [NVFP4 model card], a trained
 * projector that merges each 2 x 2 group of patches and maps the 4 x 1152 = 4608-dimensional
 * representation to the 4096-dimensional token space, 40,119,040 parameters).  The parameter
 * count fixes the structure: a LayerNorm over each patch's D features (weight and bias, 2 D),
 * then Linear r^2 D -> r^2 D with bias, then Linear r^2 D -> E with bias
 * (2*1152 + (4608*4608 + 4608) + (4608*4096 + 4096) = 40,119,040).  The activation between the
 * two Linears is not stated; this library uses the exact GELU, gelu(z) = z (1 + erf(z/sqrt 2))/2.
 *   tokens:  merged windows exactly as dsv4v_aligner_forward (r x r, row-major, zero-padded grid;
 *            a padding slot is a zero vector after the norm);
 *   x: device [P, D]; ln_w, ln_b: device fp32 [D] (LayerNorm eps = cfg->eps);
 *   w1: device [r^2 D, r^2 D], b1: device fp32 [r^2 D]; w2: device [E, r^2 D], b2: device fp32 [E];
 *   out: device [T, E], config dtype.
 * Workspace: dsv4v_patch_merger_workspace_size bytes, 256-byte aligned. */
size_t dsv4v_patch_merger_workspace_size(const dsv4v_config* cfg, const dsv4v_batch* batch);
dsv4v_status dsv4v_patch_merger_forward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                        const void* x, const float* ln_w, const float* ln_b,
                                        const void* w1, const float* b1, const void* w2,
                                        const float* b2, void* out, void* workspace,
                                        size_t ws_bytes, void* stream);

/* Patch embedding ([vision-API, DeepseekV4VisionPatchEmbed]: a linear embedding of flattened
 * RGB patches, [patches, 3, patch_h, patch_w] -> [patches, vision_dim], through its `proj`):
 * x_out[p, :] = patches[p, :] . w_proj^T (+ bias), where row p of `patches` is the patch in its
 * own (channel, row, column) order, K = 3 * patch_h * patch_w values.  The pages state neither
 * the patch size nor whether `proj` has a bias: both are arguments (bias NULL = none).
 *   patches: device [n_patches, ld_patches] (config dtype; columns >= K ignored);
 *   w_proj:  device [vision_dim, ld_w], K columns used;  bias: device fp32 [vision_dim] or NULL;
 *   x_out:   device [n_patches, vision_dim], config dtype.
 *   ld_patches / ld_w: row strides in elements (0 = K).  The bf16 path needs them to be
 *   multiples of 8 (16-byte rows for TMA; K = 588 for 14 x 14 patches, e.g. stride 592) and
 *   returns DSV4V_ERR_UNSUPPORTED otherwise; the fp32 path needs them equal to K.
 * Needs no workspace.  patch_h, patch_w in [1, 64]; all pointers 16-byte aligned. */
dsv4v_status dsv4v_patch_embed(const dsv4v_config* cfg, int64_t n_patches, int patch_h, int patch_w,
                               const void* patches, int64_t ld_patches, const void* w_proj,
                               int64_t ld_w, const float* bias, void* x_out, void* stream);

/* SwiGLU gate/up ([vision-API, DeepseekV4VisionMLP]): h = silu(y . w_gate^T) * (y . w_up^T),
 * silu(z) = z / (1 + exp(-z)).  y: device [rows, D]; h: device [rows, F]. */
dsv4v_status dsv4v_swiglu(const dsv4v_config* cfg, int64_t rows, const void* y,
                          const void* w_gate, const void* w_up, void* h, void* workspace,
                          size_t ws_bytes, void* stream);

/* x <- x + a . w^T exactly as dsv4v_linear_residual (bf16 configs only), for callers that
 * cannot allocate device memory: code that runs where cudaMalloc is not allowed (inside a
 * global-mode stream capture, on a fixed memory budget handed out at start-up, behind an
 * allocator that cannot serve library scratch).  It takes no workspace and allocates nothing:
 * the GEMM's split-tile scratch is a static device array of this library (10 MiB of partials
 * and 16384 tile counters, held by every GPU that loads the library until the process exits).
 * rows <= DSV4V_NOALLOC_MAX_ROWS; a larger call, or one whose GEMM plan needs more scratch than
 * the array holds, returns DSV4V_ERR_UNSUPPORTED without launching anything.  The first call on
 * a device looks the array's device address up (cudaGetSymbolAddress); make that first call
 * before any stream capture.  All calls on a device share the one array.  A call that is
 * accepted clears, on `stream` and just before its GEMM, the counters its plan uses; a call that
 * is refused (any error status) puts nothing on the stream.  Calls that overlap on the GPU
 * (different streams, no ordering) race on the array.  The pages describe no counterpart of
 * this call. */
#define DSV4V_NOALLOC_MAX_ROWS 65536
dsv4v_status dsv4v_linear_residual_noalloc(const dsv4v_config* cfg, int64_t rows, int k,
                                           const void* a, const void* w, void* x, void* stream);

/* Synchronises `stream` and returns the first device-side failure that a kernel of this library
 * recorded on the current device since the last call, and clears the record:
 * DSV4V_ERR_LAYOUT for pseudo-token types that do not fit the images (the bridge calls below),
 * DSV4V_ERR_TIMEOUT for any other (a bounded wait that gave up, or a CTA pair whose TMEM
 * allocations differ).  DSV4V_ERR_CUDA if the stream reports an error; else DSV4V_OK. */
dsv4v_status dsv4v_device_error(void* stream);

/* Test hook for the bounded-wait machinery: launches one tiny kernel that waits on an
 * mbarrier nothing ever signals, with a limit of `limit_ns` nanoseconds, and then records a
 * timeout exactly as the production kernels do.  Nothing faults, traps or hangs. */
dsv4v_status dsv4v_selftest_bounded_wait(uint64_t limit_ns, void* stream);

const char* dsv4v_status_string(dsv4v_status s);

/* ---------------------------------------------------------------- backward
 * The gradient of the tower ([PR], Validation: the pages train the tower and test "ragged grids
 * and backward"; no backward is printed, so each call is the chain rule through the forward
 * above).  bf16 configs only (DSV4V_ERR_UNSUPPORTED otherwise): activations and gradients are
 * bf16, norm weights and their gradients fp32, GEMMs accumulate in fp32.  Every call takes the scratch of dsv4v_backward_workspace_size and writes
 * its outputs (gradients are not accumulated into the destination). */

/* Weight gradients of one block, laid out like dsv4v_block_weights: norm1_w, norm2_w fp32 [D];
 * wqkv [3D, D], wo [D, D], w_gate [F, D], w_up [F, D], w_down [D, F] bf16.  Device pointers,
 * 16-byte aligned, written. */
typedef struct {
  float* norm1_w;
  float* norm2_w;
  void* wqkv;
  void* wo;
  void* w_gate;
  void* w_up;
  void* w_down;
} dsv4v_block_grads;

/* Bytes of device scratch every backward call below needs for this config and batch; 0 if the
 * arguments are invalid or the config is not bf16. */
size_t dsv4v_backward_workspace_size(const dsv4v_config* cfg, const dsv4v_batch* batch);

/* Gradient of the attention ([vision-API, DeepseekV4VisionAttention]; see dsv4v_attention):
 * per image and head, dv = P^T do, dS = P * (do v^T - rowsum(do * o)), dq = dS k / sqrt(hd),
 * dk = dS^T q / sqrt(hd), with P the softmax of the forward.
 *   qkv: device [P, 3D], the forward's input (q and k already rotated); out: device [P, D], the
 *   forward's output; d_out: device [P, D]; dqkv: device [P, 3D], written: the gradients with
 *   respect to the rotated q, k and to v.
 * P is rebuilt from each row's log-sum-exp, which this call recomputes with the forward
 * attention kernel (into scratch); dsv4v_block_backward takes it from its own forward
 * recompute.  Every output row is written by exactly one CTA (no atomics): the result does not
 * depend on the schedule. */
dsv4v_status dsv4v_attention_backward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                      const void* qkv, const void* out, const void* d_out,
                                      void* dqkv, void* workspace, size_t ws_bytes, void* stream);

/* Gradient of RMSNorm ([vision-API, DeepseekV4VisionRMSNorm], y = w * x * r,
 * r = 1 / sqrt(mean(x^2) + eps)): dx = r (dy * w) - x r^3 ((dy * w) . x) / D, plus d_in if
 * non-NULL (a residual gradient to add); dw = sum over rows of dy * x * r.
 *   x, dy, d_in, dx: device [P, D] (P = the batch's patches); dx may equal d_in.
 *   w: device fp32 [D]; dw: device fp32 [D], written. */
dsv4v_status dsv4v_rmsnorm_backward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                    const void* x, const float* w, const void* dy,
                                    const void* d_in, void* dx, float* dw, void* workspace,
                                    size_t ws_bytes, void* stream);

/* Gradient of one block ([vision-API, DeepseekV4VisionBlock.forward], see
 * dsv4v_block_forward) with respect to its input and its weights, for the output gradient
 * d_out.  The block's intermediates are recomputed from x; then the MLP branch, norm2, the
 * output projection, attention, the inverse rotation, the fused projection and norm1 are
 * differentiated in turn, with the residual gradients added.
 *   x: device [P, D], the block's input; d_out: device [P, D]; dx: device [P, D], written
 *   (must not overlap x or d_out); cos, sin: the rotation table of dsv4v_rope2d_table;
 *   grads: host struct of device outputs. */
dsv4v_status dsv4v_block_backward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                  const dsv4v_block_weights* weights, const float* cos,
                                  const float* sin, const void* x, const void* d_out, void* dx,
                                  const dsv4v_block_grads* grads, void* workspace,
                                  size_t ws_bytes, void* stream);

/* Gradient of the tower ([vision-API, DeepseekV4VisionTransformer.forward], see
 * dsv4v_tower_forward): the final norm's backward (if final_norm_w is non-NULL), then every
 * block's backward from the last to the first.  The caller keeps the forward's activations:
 *   layer_inputs: host array of cfg->n_layers device pointers, the input [P, D] of each block;
 *   x_last: device [P, D], the last block's output (the final norm's input; unused without a
 *   final norm); d_out: device [P, D], the gradient of the tower's output; dx: device [P, D],
 *   written; layer_grads: host array of cfg->n_layers gradient structs; d_final_norm_w: device
 *   fp32 [D], written (unused without a final norm). */
dsv4v_status dsv4v_tower_backward(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                  const dsv4v_block_weights* layers, const float* final_norm_w,
                                  const void* const* layer_inputs, const void* x_last,
                                  const void* d_out, void* dx,
                                  const dsv4v_block_grads* layer_grads, float* d_final_norm_w,
                                  void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- image-token bridge
 * [model-API, DeepseekV4Model]: the sentinel parameters image_start, image_end, image_newline
 * and image_pad; merge_image_embeddings; apply_deepseek_v4_image_visibility.
 * Pseudo-token types, one int32 per sequence position.  The pages state only -1 = text; the
 * other codes are a reading.  A span runs from an image_start to the next image_end of the
 * same sequence, and every other pseudo token must lie inside one. */
enum {
  DSV4V_TOKEN_TEXT = -1,
  DSV4V_TOKEN_IMAGE = 0,    /* takes the next aligner token of its image */
  DSV4V_TOKEN_START = 1,    /* image_start sentinel (sentinel row 0) */
  DSV4V_TOKEN_END = 2,      /* image_end sentinel (row 1) */
  DSV4V_TOKEN_NEWLINE = 3,  /* image_newline sentinel (row 2) */
  DSV4V_TOKEN_PAD = 4       /* image_pad sentinel (row 3) */
};

/* The N-layout of one image (host computation, reading adopted): image_start, then each of the
 * ceil(grid_h / r) rows of ceil(grid_w / r) aligner tokens followed by image_newline, then
 * image_end: 2 + rows * (cols + 1) types.  *length_out (if non-NULL) receives that length.
 * types_out: host int32 array of `capacity` entries, written if non-NULL.
 * DSV4V_ERR_INVALID_ARG for a grid or r below 1, or types_out with capacity below the length
 * (nothing is written then). */
dsv4v_status dsv4v_image_layout(int grid_h, int grid_w, int downsample_ratio, int32_t* types_out,
                                int64_t capacity, int64_t* length_out);

/* Bytes of device scratch that dsv4v_merge_image_embeddings and dsv4v_image_visibility need for
 * n_positions = n_seqs * seq_len positions (16 bytes per 256 positions plus 12 bytes per
 * position, each part rounded up to 256 bytes); 0 unless 1 <= n_positions < 2^31. */
size_t dsv4v_bridge_workspace_size(int64_t n_positions);

/* [model-API, DeepseekV4Model.merge_image_embeddings]: replaces every pseudo-token row of the
 * text embeddings; text rows are not touched.  Reading adopted: the image spans, in batch-major
 * order, are the batch's images in packing order; the feature positions of the j-th span take
 * image j's aligner tokens in order, and the span must hold exactly that many.
 *   token_types:  device int32 [n_seqs * seq_len], batch-major.
 *   image_tokens: device [T, E] in the config dtype (dsv4v_aligner_forward's output; T and the
 *                 per-image counts follow from cfg->downsample_ratio and the batch's grids).
 *   sentinels:    device [4, E] in the config dtype: image_start, image_end, image_newline,
 *                 image_pad.
 *   embeds:       device [n_seqs, seq_len, E] in the config dtype, updated in place; must not
 *                 overlap image_tokens or sentinels.
 * E = cfg->llm_dim; E times the element size must be a multiple of 16 bytes, and the three
 * matrices 16-byte aligned (else DSV4V_ERR_UNSUPPORTED / DSV4V_ERR_INVALID_ARG).
 * n_seqs * seq_len < 2^31.  workspace: device, 256-byte aligned, at least
 * dsv4v_bridge_workspace_size(n_seqs * seq_len) bytes.  Types that do not fit the images (an
 * unknown code, a pseudo token outside a span, an unclosed or nested span, a span whose
 * feature count differs from its image's, more or fewer spans than images) are found on the
 * device: the offending rows are left as they were, and the next dsv4v_device_error returns
 * DSV4V_ERR_LAYOUT. */
dsv4v_status dsv4v_merge_image_embeddings(const dsv4v_config* cfg, const dsv4v_batch* batch,
                                          int64_t n_seqs, int64_t seq_len,
                                          const int32_t* token_types, const void* image_tokens,
                                          const void* sentinels, void* embeds, void* workspace,
                                          size_t ws_bytes, void* stream);

/* [model-API, apply_deepseek_v4_image_visibility]: every pair of positions inside one image
 * span becomes visible (entry set to 0); every other entry is kept.
 *   token_types: device int32 [n_seqs * seq_len], batch-major.
 *   mask:        device additive mask [n_seqs, seq_len, seq_len] (the pages' [batch, 1, seq,
 *                seq]) of elem_bytes 2 (bf16 / fp16) or 4 (fp32) per entry, elem_bytes-aligned,
 *                updated in place.
 *   workspace:   device, 256-byte aligned, at least dsv4v_bridge_workspace_size(n_seqs *
 *                seq_len) bytes.
 * Types that are not well formed (see dsv4v_merge_image_embeddings) are found on the device:
 * the next dsv4v_device_error returns DSV4V_ERR_LAYOUT, and the mask may then hold zeros in
 * some rows of the malformed spans; rows of text and entries outside each row's own sequence
 * are never written. */
dsv4v_status dsv4v_image_visibility(int64_t n_seqs, int64_t seq_len, const int32_t* token_types,
                                    void* mask, int elem_bytes, void* workspace, size_t ws_bytes,
                                    void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSV4V_H */
