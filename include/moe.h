/*
 * moe.h — C ABI of libmoe.so: the forward pass of the Step-3.5-Flash sparse
 * MoE FFN layer on one NVIDIA B200 (sm_100a).
 *
 * The layer (sglang-jax issue #1367 "[Feature] Support Step 3.5 Flash",
 * section "Model configuration", MoE bullet, and section "Key difficulties",
 * item 1; llm-atlas "Step-3.5-Flash", table "Raw config fields"):
 *
 *   l   = x . W_r                       router logits, fp32 (need_fp32_gate)
 *   s   = sigmoid(l)                    fp32 scores (moe_router_activation)
 *   S   = top-k of (s + b)              the bias selects only (use_moe_router_bias)
 *   g_j = 3 * s_{S_j} / sum_j s_{S_j}   bias-free, renormalised (norm_expert_weight),
 *                                       scaled (moe_router_scaling_factor 3)
 *   out = sum_j g_j * f_{S_j}(x) + f_shared(x)
 *   f(x) = (silu(gate) * up) . W_down,  gate = x . W_gate, up = x . W_up,
 *          with the optional clamp gate = min(gate, L), up = clip(up, -L, L)
 *          (swiglu_limits / swiglu_limits_shared; L = 0 means no clamp).
 *
 * Selection order and ties: descending s + b, equal scores to the lower
 * expert index.  The shared expert has no gate and weight 1.
 *
 * Arithmetic: the router, the scores, the selection and the gate weights are
 * fp32 on the CUDA cores (from 512 bf16 tokens the logits are first
 * approximated on the tensor cores and every expert near the selection
 * boundary is recomputed in fp32).  The expert GEMMs follow weight_dtype:
 *  - bf16 (and FP8) weights: bf16 x bf16 with fp32 accumulation.  fp32 x is
 *    rounded to bf16 (round to nearest even) on the way in, h = SwiGLU(...)
 *    and each expert's weighted output row are rounded to bf16, and the
 *    k + 1 rows of a token are summed in fp32 and rounded once to the output
 *    dtype.  Error budget: each bf16 rounding is a relative error of at most
 *    2^-9; with independent rounding errors over K-term sums the output's
 *    relative Frobenius error stays near 2^-9 times a small constant (~3e-3
 *    measured at the full layer against the fp64 definition).
 *  - fp32 weights (weight_dtype MOE_F32): the fp32 expert path.  Every GEMM
 *    operand (weights, x, h) is split into two tf32 terms v = v_hi + v_lo
 *    (v_hi = v rounded to tf32, v_lo = v - v_hi), and the tf32 tensor cores
 *    accumulate w_hi x_hi + w_lo x_hi + w_hi x_lo in fp32: each product to
 *    within ~2^-21 of fp32's.  h and the output rows stay fp32 and are summed
 *    in fp32.  Measured against the fp64 definition: ~6e-6 relative
 *    Frobenius error on the tiny fp32 layer, dominated by the tensor cores'
 *    fp32 accumulation, which behaves like truncation at every MMA step and
 *    so grows with K (~1e-4 expected at H = 4096).  Costs: 8 bytes of device memory
 *    per expert weight and three MMA passes; always on one-SM tiles (no CTA
 *    pairs, no fused forward).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers unless the name says _host.
 *    They are owned by the caller; the library never frees or keeps them past
 *    the call, except that a layer handle owns its own packed weight copy.
 *  - Layouts are row-major: x [T, H], out [T, H], router_w [H, E],
 *    router_bias [E], w_gate / w_up [E, H, I], w_down [E, I, H],
 *    sh_gate / sh_up [H, Is], sh_down [Is, H].
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Work is enqueued on it; no entry point synchronises the host
 *    unless its comment says so.
 *  - Every entry point returns a moe_status_t.  Arguments are checked on the
 *    host first; on any error nothing is enqueued and outputs are untouched.
 *  - T = 0 is a valid no-op.
 */
#ifndef SPARSE_MOE_LAYER_GEMM_B200_MOE_H
#define SPARSE_MOE_LAYER_GEMM_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,     /* null pointer, negative size, bad enum */
  MOE_ERR_UNSUPPORTED = 2,     /* valid but outside what the kernels handle */
  MOE_ERR_WORKSPACE = 3,       /* workspace missing, too small or misaligned */
  MOE_ERR_CUDA = 4,            /* a CUDA runtime call failed */
  MOE_ERR_DEVICE_TIMEOUT = 5,  /* a kernel gave up a bounded wait (device error word) */
  MOE_ERR_NOT_LOADED = 6       /* moe_forward before moe_load_weights */
} moe_status_t;

/* MOE_FP8_E4M3: expert weights only (weight_dtype), loaded with
 * moe_load_weights_fp8.  The pages list FP8 official weights for the model
 * (sglang-jax issue #1367, section "Model configuration", "Official weights")
 * without a format; the one taken here is E4M3FN codes (sign, 4-bit exponent
 * with bias 7, 3-bit mantissa, no infinities, S.1111.111 = NaN) with one fp32
 * scale per output feature: w[k][n] = value(code[k][n]) * scale[n]. */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_FP8_E4M3 = 2 } moe_dtype_t;

/* Layer configuration.  Field names follow the model's config fields
 * (llm-atlas "Step-3.5-Flash", "Raw config fields").
 * Supported: hidden % 128 == 0, 1 <= hidden <= 16384; 1 <= num_experts <= 1024;
 * 1 <= top_k <= min(num_experts, 32); 1 <= intermediate <= 8192;
 * shared_intermediate == intermediate; act_dtype in {F32, BF16}; weight_dtype
 * in {F32, BF16, FP8_E4M3};
 * routed_scaling_factor finite; swiglu limits >= 0 (0 = no clamp). */
typedef struct {
  int hidden;                  /* H: hidden_size, 4096 */
  int num_experts;             /* E: moe_num_experts, 288 */
  int top_k;                   /* k: moe_top_k, 8 */
  int intermediate;            /* I: moe_intermediate_size, 1280 */
  int shared_intermediate;     /* Is: share_expert_dim, 1280 */
  int norm_expert_weight;      /* 1: renormalise the top-k scores */
  float routed_scaling_factor; /* 3.0 */
  int use_router_bias;         /* 1: add router_bias to the scores for selection */
  float swiglu_limit;          /* routed experts' clamp, 0 = none */
  float swiglu_limit_shared;   /* shared expert's clamp, 0 = none */
  int act_dtype;               /* moe_dtype_t of x and out */
  int weight_dtype;            /* moe_dtype_t of the expert weights passed to load */
} moe_config_t;

typedef struct moe_layer moe_layer_t;

/* Optional routing outputs of moe_forward (device pointers, caller-owned;
 * any field may be NULL).  topk_idx [T, k] int32 (descending s + b),
 * topk_w [T, k] fp32 gate weights, counts [E] int32 pairs per expert,
 * offsets [E + 1] int32 exclusive prefix of counts, perm [T * k] int32 pair
 * ids t * k + j grouped by expert, ascending t within an expert, logits
 * [T, E] fp32 router logits x . W_r as used for the selection. */
typedef struct {
  int32_t* topk_idx;
  float* topk_w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  float* logits;
} moe_routing_t;

/* Host-only check of a configuration; no CUDA call.  Returns MOE_OK,
 * MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED. */
int moe_config_check(const moe_config_t* cfg);

/* Creates a layer on the current CUDA device.  Allocates the packed weight
 * copy (3 * (E + 1) * H * round_up(I, 128) bf16; for fp32 weights two fp32
 * values each; for FP8 weights one byte each plus (E + 1) * (2 *
 * round_up(I, 128) + H) fp32 scales; plus the router) and a small device
 * status word.  *out receives the handle (NULL on
 * error). */
int moe_create(const moe_config_t* cfg, moe_layer_t** out);

/* Expert parallelism: a layer holding only the routed experts
 * [expert_first, expert_first + expert_count) of the configuration's E (and
 * the shared expert if with_shared is 1).  Routing still covers all E
 * experts (the router weight is loaded whole); moe_forward then computes only
 * this shard's experts for the pairs that selected them (and the shared
 * expert if held) and writes their weighted sum to out: summed over shards
 * that cover every expert once (and the shared expert once), e.g. by an
 * all-reduce across the GPUs that hold them, it is the layer's output.  The
 * load entry points take the full [E, ...] expert tensors and pick the
 * shard's slice.  With a shard, moe_routing_t's counts [expert_count] and
 * offsets [expert_count + 1] are the shard's, perm lists its pairs first.
 * Returns MOE_ERR_INVALID_ARG for an empty or out-of-range expert range or
 * with_shared not 0/1.  moe_create(cfg) is moe_create_shard(cfg, 0, E, 1). */
int moe_create_shard(const moe_config_t* cfg, int expert_first, int expert_count,
                     int with_shared, moe_layer_t** out);

/* Copies the weights into the layer's packed layout on `stream` (K-major
 * weight rows; gate and up interleaved in blocks of 128 rows): bf16, or for
 * fp32 expert weights the fp32 expert path's two tf32 terms of each weight
 * (see the arithmetic note at the top).  router_w [H, E] and router_bias [E]
 * are fp32 and kept fp32; router_bias may be NULL (zero bias).  The expert
 * pointers have the config's weight_dtype (F32 or BF16; a layer created with
 * MOE_FP8_E4M3 weights returns MOE_ERR_INVALID_ARG: it loads through
 * moe_load_weights_fp8).  The caller's buffers may be freed once `stream` has
 * passed this call. */
int moe_load_weights(moe_layer_t* layer, const float* router_w, const float* router_bias,
                     const void* w_gate, const void* w_up, const void* w_down,
                     const void* sh_gate, const void* sh_up, const void* sh_down,
                     void* stream);

/* moe_load_weights for an expert shard (moe_create_shard) whose caller holds
 * only the shard's own experts: w_gate, w_up [expert_count, H, I] and w_down
 * [expert_count, I, H] start at the shard's first expert (moe_load_weights
 * takes the whole [E, ...] tensors and skips to it).  sh_gate / sh_up /
 * sh_down may be NULL when the shard holds no shared expert.  router_w and
 * router_bias are the whole layer's (every shard routes over all experts).
 * Lets each rank of an expert-parallel layer load 1/N of the expert bytes.
 * bf16 / fp32 weights (a layer created with MOE_FP8_E4M3 returns
 * MOE_ERR_INVALID_ARG). */
int moe_load_shard_weights(moe_layer_t* layer, const float* router_w, const float* router_bias,
                           const void* w_gate, const void* w_up, const void* w_down,
                           const void* sh_gate, const void* sh_up, const void* sh_down,
                           void* stream);

/* FP8 expert weights (layer created with weight_dtype MOE_FP8_E4M3): the
 * codes in the layouts of moe_load_weights, one uint8 E4M3FN code per weight
 * (w_gate / w_up [E, H, I], w_down [E, I, H], sh_gate / sh_up [H, I],
 * sh_down [I, H]), and their fp32 scales per output feature: s_gate / s_up
 * [E, I], s_down [E, H], sh_s_gate / sh_s_up [I], sh_s_down [H].  NaN codes
 * (0x7F, 0xFF) are not valid weights.  The codes are kept as bytes (no bf16
 * copy); the expert GEMMs expand them to bf16 in shared memory, exactly, and
 * multiply each output feature's accumulator by its scale.  Router as in
 * moe_load_weights.  Returns MOE_ERR_INVALID_ARG for a NULL pointer or a
 * layer whose weight_dtype is not MOE_FP8_E4M3.  Device pointers, caller
 * owned, free once `stream` has passed this call. */
int moe_load_weights_fp8(moe_layer_t* layer, const float* router_w, const float* router_bias,
                         const uint8_t* w_gate, const uint8_t* w_up, const uint8_t* w_down,
                         const float* s_gate, const float* s_up, const float* s_down,
                         const uint8_t* sh_gate, const uint8_t* sh_up, const uint8_t* sh_down,
                         const float* sh_s_gate, const float* sh_s_up, const float* sh_s_down,
                         void* stream);

/* E4M3FN codes -> bf16 values (uint16 bit patterns) on `stream`, through the
 * same routine the FP8 expert GEMMs expand their weights with (every finite
 * code is exactly a bf16 value; NaN codes give +-480, see
 * moe_load_weights_fp8).  codes and out are device pointers, 16-byte
 * aligned; n % 4 == 0 (MOE_ERR_INVALID_ARG otherwise); n = 0 is a no-op. */
int moe_decode_e4m3(const uint8_t* codes, size_t n, uint16_t* out, void* stream);

/* Device workspace bytes moe_forward needs for T tokens (caller allocates,
 * 256-byte aligned).  Host-only. */
int moe_workspace_size(const moe_layer_t* layer, int T, size_t* bytes);

/* The layer forward: out [T, H] (act_dtype) from x [T, H] (act_dtype).
 * Stream-ordered, no host synchronisation, capturable in a CUDA graph once
 * the weights are loaded.  `routing` may be NULL.  x and out must not alias. */
int moe_forward(moe_layer_t* layer, const void* x, int T, void* out,
                void* workspace, size_t ws_bytes, void* stream,
                const moe_routing_t* routing);

/* Execution paths of moe_forward.
 *  MOE_PATH_MULTI: one kernel per stage (router, top-k, sort, gather,
 *    gate|up GEMM, down GEMM, combine: 7 to 10 launches).
 *  MOE_PATH_FUSED: the whole layer in one persistent kernel (the pages'
 *    FusedEPMoE backend, sglang-jax issue #1367, section "Reuse map" and the
 *    sub-issue "FusedEPMoE performance backend switch"): routing, sort,
 *    both expert GEMMs and the combine as phases of one launch, the down
 *    tiles starting as soon as their token block's gate|up tiles are done,
 *    the token rows read straight from x (no gathered copy).  Same results,
 *    bit for bit, as the multi-launch path.  Eligible for bf16 x and bf16
 *    weights, T >= 2048, hidden / 128 even, num_experts <= 288, a whole layer
 *    (not a shard); otherwise moe_forward takes the multi-launch path.  Its
 *    grid-wide barriers need every CTA of the launch resident at once (one
 *    CTA pair per two SMs): kernels that occupy SMs on other streams for
 *    seconds make its bounded waits expire (MOE_ERR_DEVICE_TIMEOUT through
 *    moe_get_device_error) rather than hang.
 *  MOE_PATH_AUTO (default): the fused path where it is eligible and measured
 *    faster, else the multi-launch path. */
#define MOE_PATH_AUTO 0
#define MOE_PATH_MULTI 1
#define MOE_PATH_FUSED 2

/* Selects the path of the following forwards (MOE_ERR_INVALID_ARG for an
 * unknown path).  Host-only. */
int moe_set_path(moe_layer_t* layer, int path);

/* The path a forward of T tokens takes with the layer's current setting:
 * MOE_PATH_MULTI or MOE_PATH_FUSED (0 for a NULL layer or T <= 0). */
int moe_forward_path(const moe_layer_t* layer, int T);

/* Self-check of the fused path's bounded waits (fault detection without a
 * fault): one fused forward of x [T, H] into out (T, the layer and the
 * workspace as for moe_forward on the fused path) in which no down-projection
 * tile can ever become ready, and every bounded wait of the kernel (the
 * readiness counters, the grid barriers, the mbarriers) gives up after
 * limit_us microseconds (1 .. 10,000,000).  The down tiles' waits expire,
 * every role of the kernel winds down and frees its tensor memory, and the
 * timeout bit is set in the layer's device status word.  Synchronises the
 * device, reads and clears the word into *device_status (if not NULL).
 * Returns MOE_OK when exactly the timeout bit (1) was reported,
 * MOE_ERR_UNSUPPORTED when the fused path does not apply to this layer and T,
 * MOE_ERR_INVALID_ARG / MOE_ERR_WORKSPACE / MOE_ERR_NOT_LOADED as
 * moe_forward, MOE_ERR_CUDA otherwise.  out's contents are undefined
 * afterwards. */
int moe_check_fused_timeout(moe_layer_t* layer, const void* x, int T, void* out,
                            void* workspace, size_t ws_bytes, int limit_us,
                            int* device_status);

/* Workspace bytes for moe_forward_host and moe_forward_host_async:
 * moe_workspace_size plus two device staging slots for x and out. */
int moe_workspace_size_host(const moe_layer_t* layer, int T, size_t* bytes);

/* The forward from and to HOST buffers: copies x_host to the device, runs
 * moe_forward, copies the result to out_host, all on `stream`, then
 * synchronises `stream` before returning.  Pinned host memory makes the
 * copies asynchronous DMA; pageable memory also works. */
int moe_forward_host(moe_layer_t* layer, const void* x_host, int T, void* out_host,
                     void* workspace, size_t ws_bytes, void* stream);

/* The same for a stream of batches, pipelined: enqueues the copy of x_host
 * into one of two device staging slots (alternating per call), the forward
 * on `stream`, and the copy of the result to out_host, and returns without
 * waiting.  The copies run on two streams owned by the layer, ordered with
 * `stream` by events, so a call's input copy overlaps the previous call's
 * forward and its output copy the next call's.  Host buffers must be pinned
 * (page-locked) and left untouched until the call's copies are done: after
 * moe_forward_host_join(layer, s) and a synchronisation of s.  Calls of one
 * layer must come from one host thread, on one stream, with one workspace
 * (of moe_workspace_size_host bytes for the largest T); a call with another
 * T than the previous one first waits for every earlier call's copies. */
int moe_forward_host_async(moe_layer_t* layer, const void* x_host, int T, void* out_host,
                           void* workspace, size_t ws_bytes, void* stream);

/* Makes `stream` wait until the output copies of every
 * moe_forward_host_async call issued so far are done (no host wait). */
int moe_forward_host_join(moe_layer_t* layer, void* stream);

/* Synchronises the device, then reads and clears the layer's device status
 * word: *device_err = 0 when no kernel reported a problem, otherwise a bit
 * mask (1 = a bounded wait timed out in a GEMM kernel).  Returns
 * MOE_ERR_DEVICE_TIMEOUT when the word was non-zero. */
int moe_get_device_error(moe_layer_t* layer, int* device_err);

/* Self-check of the bounded waits every kernel uses (fault detection
 * without a fault): launches one CTA on the current device whose wait on a
 * barrier that nothing signals gives up after `limit_us` microseconds
 * (1 .. 10,000,000), sets the timeout bit (1) of a device status word and
 * returns.  Synchronises the device.  *device_status (if not NULL) receives
 * the word.  Returns MOE_OK when the wait gave up and reported exactly the
 * timeout bit, MOE_ERR_INVALID_ARG for a bad limit, MOE_ERR_CUDA otherwise.
 * Allocates and frees 4 bytes of device memory. */
int moe_check_wait_timeout(int limit_us, int* device_status);

/* Static description of a status code. */
const char* moe_status_string(int status);

/* Frees the layer and its device memory.  NULL is ignored.  Synchronises
 * the device first. */
void moe_destroy(moe_layer_t* layer);

/* Stages of one forward, in launch order, for the stage timers below:
 * 0 router logits, 1 top-k and gate weights, 2 counting sort (3 kernels),
 * 3 gather of the input rows, 4 grouped gate|up GEMM + SwiGLU,
 * 5 grouped down GEMM x gate weight, 6 combine.  A forward on the fused path
 * is one kernel: its whole time is recorded as stage 0, the others as 0. */
#define MOE_NUM_STAGES 7

/* Kernel launches one moe_forward makes for T tokens (0 for T = 0). */
int moe_kernel_launches(const moe_layer_t* layer, int T);

/* Per-stage device timing.  With capacity > 0 each following moe_forward
 * records CUDA events around its stages on its own stream, for up to
 * `capacity` forwards (later forwards are not recorded); capacity 0 turns
 * timing off and frees the events.  Host-side setup only. */
int moe_set_stage_timing(moe_layer_t* layer, int capacity);

/* Waits for the recorded events, writes the summed milliseconds of each stage
 * over the recorded forwards to ms[0 .. n_stages-1] (n_stages <=
 * MOE_NUM_STAGES) and their number to *n_forwards, then starts a new
 * recording window of the same capacity. */
int moe_get_stage_times(moe_layer_t* layer, float* ms, int n_stages, int* n_forwards);

/* One call with the layer's argument list: creates a layer, loads the
 * weights, allocates a workspace, runs the forward on `stream`, synchronises
 * and frees everything.  Convenient for a single forward; for repeated calls
 * use create / load / forward.  Allocates device memory (cudaMalloc).
 * weight_dtype MOE_FP8_E4M3 returns MOE_ERR_UNSUPPORTED (this argument list
 * has no scales; use create / moe_load_weights_fp8 / forward). */
int moe_forward_oneshot(const void* x, const float* router_w, const float* router_bias,
                        const void* w_gate, const void* w_up, const void* w_down,
                        const void* sh_gate, const void* sh_up, const void* sh_down,
                        int T, int H, int E, int k, int I, float scale,
                        float swiglu_limit, float swiglu_limit_shared,
                        int act_dtype, int weight_dtype, void* out, void* stream);

/* Routing without any device allocation: router logits x . W_r (fp32),
 * sigmoid scores, top-k of score + router_bias (descending, ties to the lower
 * index), and the gate weights scale * s / sum(s) of the selected bias-free
 * scores (plain scale * s when norm_expert_weight is 0).  The source pages
 * have no counterpart of this entry point: it exists for callers that cannot
 * call cudaMalloc, such as code running under CUDA-graph capture, runtimes
 * that own all of HBM through their own pool, or latency-critical loops where
 * an allocation could synchronise the device.  It needs no layer handle and
 * no workspace.
 *
 * x [T, H] (act_dtype, 16-byte aligned), router_w [H, E] fp32, router_bias
 * [E] fp32 or NULL; outputs topk_idx [T, k] int32 and topk_w [T, k] fp32, all
 * device pointers owned by the caller.  It runs the router on the CUDA cores
 * with the K split moe_forward uses there (below 512 tokens, or fp32 x), and
 * gives identical results whenever T * E * H / 128 <= 1,048,576 (else it
 * uses fewer splits).  From 512 bf16 tokens moe_forward runs the router on
 * the tensor cores; the two then agree to fp32 rounding (the selection can
 * differ only on tokens whose k-th and (k+1)-th scores are within ~1e-6).
 *
 * Scratch: a 4 MiB static device array inside the library (1,048,576 fp32
 * partial logits), held on a GPU from the first call on that device (module
 * loading may be lazy) until the process exits.  T * E must not exceed
 * 1,048,576 (MOE_ERR_UNSUPPORTED otherwise).  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  The
 * address is kept per device together with the id of the context it was
 * taken in; a call whose current context differs (for instance after a
 * cudaDeviceReset) looks it up again, so that call, too, should come before
 * any capture.  Every call uses the same array, so calls that may overlap on
 * the GPU (different streams, or different host threads) race and must be
 * serialised by the caller.  No cudaMalloc, cudaFree or other allocating
 * routine is called. */
int moe_route_static(const void* x, int act_dtype, const float* router_w,
                     const float* router_bias, int T, int H, int E, int k,
                     int norm_expert_weight, float routed_scaling_factor,
                     int32_t* topk_idx, float* topk_w, void* stream);

/* ---------------------------------------------------------------- dense MLP
 * The dense SwiGLU MLP of the model's first three decoder layers
 * (sglang-jax issue #1367, section "Model configuration", MLP bullet: the
 * first 3 layers are dense, intermediate 11264; llm-atlas "Step-3.5-Flash",
 * table "Raw config fields", intermediate_size 11264):
 *
 *   out = (silu(min(x.W_gate, L)) * clip(x.W_up, -L, L)) . W_down
 *
 * (L = 0: no clamp), computed by the MoE layer's expert GEMMs with one group
 * of all T rows.  Same conventions as the MoE entry points: device pointers,
 * caller-owned; x [T, H] and out [T, H] in act_dtype; w_gate, w_up [H, I],
 * w_down [I, H] in weight_dtype (fp32 weights take the fp32 expert path of
 * the MoE layer: tf32 tensor cores over the two-term split, h fp32, one-SM
 * tiles at every T);
 * stream-ordered, no host synchronisation in the forward; every argument is
 * checked on the host and nothing is enqueued on error. */
typedef struct moe_dense moe_dense_t;

/* Supported: hidden % 128 == 0, hidden <= 16384; 1 <= intermediate <=
 * 32768; act_dtype in {F32, BF16}; weight_dtype in {F32, BF16}
 * (MOE_FP8_E4M3 returns MOE_ERR_UNSUPPORTED); swiglu_limit finite, >= 0. */
typedef struct {
  int hidden;          /* H: hidden_size, 4096 */
  int intermediate;    /* I: intermediate_size, 11264 */
  float swiglu_limit;  /* clamp, 0 = none */
  int act_dtype;       /* moe_dtype_t of x and out */
  int weight_dtype;    /* moe_dtype_t of the weights passed to load */
} moe_dense_config_t;

/* Host-only check of a configuration; no CUDA call. */
int moe_dense_config_check(const moe_dense_config_t* cfg);

/* Creates the layer on the current device: packed weights (3 * H *
 * round_up(I, 128) elements: bf16, or two fp32 terms each for fp32 weights)
 * and a device status word. */
int moe_dense_create(const moe_dense_config_t* cfg, moe_dense_t** out);

/* Copies the weights into the packed layout on `stream` (the caller's
 * buffers may be freed once `stream` has passed this call). */
int moe_dense_load_weights(moe_dense_t* layer, const void* w_gate, const void* w_up,
                           const void* w_down, void* stream);

/* Device workspace bytes moe_dense_forward needs for T tokens (256-byte
 * aligned, caller-allocated).  Host-only. */
int moe_dense_workspace_size(const moe_dense_t* layer, int T, size_t* bytes);

/* out [T, H] from x [T, H]; x and out must not alias; T = 0 is a no-op.
 * From 1 to 128 tokens with hidden % 256 == 0 the forward is one persistent
 * launch whose CTAs synchronise through running counters owned by the layer
 * (never cleared between forwards): the forwards of one layer must then run
 * on the device in the order they were issued (one stream, or streams
 * ordered by events).  The counters' targets are derived on the device, so
 * the forward may be captured in a CUDA graph and replayed.  The result
 * depends only on x's own rows (the same row gives the same output in any
 * batch of up to 128 tokens). */
int moe_dense_forward(moe_dense_t* layer, const void* x, int T, void* out,
                      void* workspace, size_t ws_bytes, void* stream);

/* As moe_get_device_error, for the dense layer's status word.  After a
 * device error it also clears the layer's forward counters (the aborted
 * launch left them short), so later forwards start from a clean state. */
int moe_dense_get_device_error(moe_dense_t* layer, int* device_err);

/* Frees the layer (synchronises the device first).  NULL is ignored. */
void moe_dense_destroy(moe_dense_t* layer);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_MOE_LAYER_GEMM_B200_MOE_H */
