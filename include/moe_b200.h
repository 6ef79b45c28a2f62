/*
 * moe_b200.h — C ABI of the B200 (sm_100a) forward pass of the biased-sigmoid-routed
 * Mixture-of-Experts FFN layer of Step-3.5-Flash / Step-5-Preview.
 *
 * The layer ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪",
 * config keys from section "Step3p5Config配置项全解"):
 *   logits  = x · Wr^T                      computed in FP32 (the FP32 gate)
 *   s       = sigmoid(logits)
 *   ids     = top-k of (s + router_bias)    bias used for selection only; ties to the
 *                                           lower expert index; a NaN score ranks last
 *   w_j     = scale · s_j / Σ_j s_j         (norm_expert_weight; no epsilon; if the sum
 *                                           is 0 every weight is scale/k), or scale · s_j
 *   y       = Σ_j w_j · SwiGLU_{ids_j}(x; L_routed) + SwiGLU_shared(x; L_shared)
 *   SwiGLU(x; L) = Wd · (min(silu(g), L) ⊙ clamp(u, −L, L)), g = Wg·x, u = Wu·x; L = 0: no clip.
 *
 * Conventions for every entry point:
 *  - All array arguments are DEVICE pointers on the current CUDA device, allocated and
 *    owned by the caller. The library never allocates, frees or synchronises; it only
 *    enqueues kernels (and, where stated, a memset) on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).
 *  - bf16 arrays are passed as uint16_t bit patterns. Matrices are row-major with the
 *    reduction dimension innermost (PyTorch [out, in]).
 *  - Argument checks run on the host before anything is enqueued; on any error nothing
 *    is enqueued and the outputs are untouched. MOE_ERR_INVALID_ARG: NULL pointer, bad
 *    sizes or k outside [1, min(E, 32)]. MOE_ERR_UNSUPPORTED: H not a multiple of 128,
 *    I or Is not a multiple of 64, E > 512, a bf16/fp32 array not 16-byte aligned, or
 *    sizes whose index arithmetic would overflow 32-bit row counts. MOE_ERR_WORKSPACE:
 *    ws_bytes below moe_workspace_size(). MOE_ERR_CUDA: a launch failed (the CUDA error
 *    is left for cudaGetLastError()).
 *  - Device-side waits are bounded; a wait that expires sets a device error word that
 *    moe_check_device() reports as MOE_ERR_TIMEOUT. Kernels never trap.
 *  - Debug build (libmoe_b200_debug.so, compiled with MOE_DEBUG): every index the kernels
 *    read from device data (expert ids, slots, tile-table entries, destination rows) is
 *    range-checked before use; a failed check sets a bit of the device error word, the
 *    access is clamped into range or skipped (no fault, results then meaningless), and
 *    moe_check_device() reports MOE_ERR_DEVICE_BOUNDS. The release build compiles the
 *    checks out.
 *  - T = 0 is valid: after the descriptor check the call returns MOE_OK without
 *    enqueueing anything, and the array pointers may then be NULL.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_WORKSPACE = 3,
    MOE_ERR_CUDA = 4,
    MOE_ERR_TIMEOUT = 5,
    MOE_ERR_DEVICE_BOUNDS = 6
} moe_status_t;

/* One MoE layer call. Field names follow Step3p5Config ("Step3p5Config配置项全解"):
 * E = moe_num_experts, k = moe_top_k, I = moe_intermediate_size, Is = share_expert_dim,
 * scale = moe_router_scaling_factor, norm_expert_weight, limit_routed =
 * swiglu_limits[layer], limit_shared = swiglu_limits_shared[layer] (0 = no clip).
 * deterministic = 1 selects the fixed-order combine (moe_combine) instead of fp32
 * atomic accumulation into y; both give the same value up to fp32 summation order. */
typedef struct {
    int32_t T;  /* tokens */
    int32_t H;  /* hidden size */
    int32_t E;  /* routed experts */
    int32_t k;  /* experts per token */
    int32_t I;  /* routed expert intermediate size */
    int32_t Is; /* shared expert intermediate size */
    float scale;
    int32_t norm_expert_weight;
    float limit_routed;
    float limit_shared;
    int32_t deterministic;
} moe_layer_desc;

/* Human-readable name of a status code (static string). */
MOE_API const char *moe_status_string(int status);

/* Bytes of device workspace that moe_expert_ffn and moe_forward need for `desc`
 * (written to *bytes). The workspace holds the permuted activations, the hidden
 * SwiGLU activations, per-slot weights, the tile table and (moe_forward) the routing
 * tables. Its contents need not be initialised. */
MOE_API moe_status_t moe_workspace_size(const moe_layer_desc *desc, size_t *bytes);

/* Router ("MoE共享专家、sigmoid 路由与激活裁剪": FP32 gate, sigmoid, router_bias for selection
 * only, top-k, normalisation, scaling; index clamp to [0, E-1]).
 *   x [T, H] bf16, Wr [E, H] bf16, bias [E] fp32 (inputs, read-only)
 *   topk_idx [T, k] int32: selected experts in rank order (biased score descending,
 *                          ties to the lower index)
 *   topk_w   [T, k] fp32:  routing weights (from the unbiased scores)
 *   margin   [T] fp32 or NULL: (k-th biased score) - ((k+1)-th), +inf when k = E. */
MOE_API moe_status_t moe_router(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                        const float *bias, int32_t *topk_idx, float *topk_w, float *margin,
                        void *stream);

/* Token -> slot permutation, bit-exact and deterministic: per-expert histogram,
 * exclusive scan, and a scatter stable in token order. Group E is the shared expert and
 * holds every token in order.
 *   topk_idx [T, k] int32 (input; ids outside [0, E-1] are clamped)
 *   counts [E+1]: tokens per group (counts[E] = T)
 *   offsets [E+2]: exclusive scan of counts (offsets[E] = T*k, offsets[E+1] = T*k + T)
 *   perm_token [T*k + T]: token of each slot; slots of group e are
 *              [offsets[e], offsets[e+1]) in ascending token order
 *   slot_of [T, k]: slot of (token, rank j); the inverse of perm_token on routed slots. */
MOE_API moe_status_t moe_permute(const moe_layer_desc *desc, const int32_t *topk_idx, int32_t *counts,
                         int32_t *offsets, int32_t *perm_token, int32_t *slot_of, void *stream);

/* Routed and shared expert FFNs with the clipped SwiGLU ("MoE共享专家、sigmoid 路由与激活裁剪":
 * routed_moe(x) + shared_expert(x), make_concatenated_gated_activation_fn(silu, limit)).
 *   x [T, H] bf16; topk_w [T, k] fp32; offsets, perm_token, slot_of from moe_permute
 *   W_gate_up [E, 2I, H] bf16 (rows [0, I) gate, [I, 2I) up); W_down [E, H, I] bf16
 *   Wsh_gate_up [2Is, H] bf16; Wsh_down [H, Is] bf16
 *   out: deterministic = 0 -> y [T, H] fp32, overwritten (zeroed, then accumulated);
 *        deterministic = 1 -> o_perm [T*k + T, H] fp32: row slot_of[t, j] holds
 *        topk_w[t, j] * expert output, row T*k + t holds the shared expert output;
 *        moe_combine then sums them in a fixed order.
 *   ws, ws_bytes: workspace of at least moe_workspace_size() bytes. */
MOE_API moe_status_t moe_expert_ffn(const moe_layer_desc *desc, const uint16_t *x, const float *topk_w,
                            const int32_t *offsets, const int32_t *perm_token,
                            const int32_t *slot_of, const uint16_t *W_gate_up,
                            const uint16_t *W_down, const uint16_t *Wsh_gate_up,
                            const uint16_t *Wsh_down, float *out, void *ws, size_t ws_bytes,
                            void *stream);

/* Fixed-order combine: y[t] = Σ_{j<k} o_perm[slot_of[t, j]] + o_perm[T*k + t], summed in
 * rank order, then the shared row. o_perm [T*k + T, H] fp32, slot_of [T, k], y [T, H]
 * fp32 (overwritten). */
MOE_API moe_status_t moe_combine(const moe_layer_desc *desc, const float *o_perm, const int32_t *slot_of,
                         float *y, void *stream);

/* The whole layer: moe_router -> moe_permute -> moe_expert_ffn (-> moe_combine when
 * deterministic). y [T, H] fp32 is overwritten. topk_idx_out / topk_w_out ([T, k]) may be
 * NULL; when given they receive the routing. */
MOE_API moe_status_t moe_forward(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                         const float *bias, const uint16_t *W_gate_up, const uint16_t *W_down,
                         const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down, float *y,
                         int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                         void *stream);

/* The layer with the routing supplied by the caller instead of computed: rollout routing
 * replay, where a trainer replays the expert choices its rollout engine made (miles
 * Step-5-Preview recipe page, sections 5.2 "--use-rollout-routing-replay" and 5.4, which
 * needs the engine's materialised top-k ids), and the fake balanced static expert routing
 * of the NeMo AutoModel Step-5-Preview benchmark setup. moe_permute -> moe_expert_ffn
 * (-> moe_combine when deterministic).
 *   topk_idx [T, k] int32 (ids outside [0, E-1] are clamped; an id may repeat within a token,
 *   each slot then adds its own weighted copy), topk_w [T, k] fp32 routing weights, used as
 *   given (no normalisation or scaling). Other arguments as in moe_forward. */
MOE_API moe_status_t moe_forward_with_ids(const moe_layer_desc *desc, const uint16_t *x, const int32_t *topk_idx,
                                  const float *topk_w, const uint16_t *W_gate_up, const uint16_t *W_down,
                                  const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down, float *y, void *ws,
                                  size_t ws_bytes, void *stream);

/* moe_forward with FP8 E4M3 routed experts: the checkpoint format of the miles
 * Step-5-Preview page, section 1 ("FP8 checkpoint"), routed experts in FP8 E4M3 with one
 * scale per 128x128 block, dequantized on load; the shared expert stays BF16.
 *   W_gate_up_q [E, 2I, H] uint8 E4M3 codes (rows [0, I) gate, [I, 2I) up),
 *   W_gate_up_scale [E, 2I/128, H/128] fp32, W_down_q [E, H, I] uint8,
 *   W_down_scale [E, H/128, I/128] fp32: weight[r][c] = e4m3(q[r][c]) * scale[r/128][c/128].
 * The kernels stream the codes (half the weight bytes of BF16). Decode-sized calls (T * k <=
 * 16 * E) with H % 256 == 0 and I, Is % 128 == 0 feed the codes unchanged to the FP8 tensor
 * cores: each block scale, together with a power of two per token row taken from the row's
 * largest |x| (or |h|), multiplies the token operand, which is split into two E4M3 parts
 * (hi + lo, about 8 significant bits, the precision of a bf16 operand). Other calls turn the
 * codes into bf16(e4m3 * scale) in tensor memory for the BF16 tensor-core MMA, so a
 * dequantized weight carries one bf16 rounding (relative 2^-9) besides the BF16 path's
 * arithmetic. Every other
 * argument, the workspace (moe_workspace_size covers both formats) and the results are
 * those of moe_forward. Requires I % 128 == 0 (MOE_ERR_UNSUPPORTED otherwise); code arrays
 * 16-byte aligned, scale arrays 4-byte aligned; the library reads the weights only. */
MOE_API moe_status_t moe_forward_fp8(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                                     const float *bias, const uint8_t *W_gate_up_q, const float *W_gate_up_scale,
                                     const uint8_t *W_down_q, const float *W_down_scale,
                                     const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down, float *y,
                                     int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                                     void *stream);

/* Device workspace of moe_forward_host: moe_workspace_size(desc) plus two [T, H] bf16 input
 * and two [T, H] fp32 output staging buffers. */
MOE_API moe_status_t moe_host_workspace_size(const moe_layer_desc *desc, size_t *bytes);

/* moe_forward (or moe_forward_fp8) over n_batches batches of T tokens that live in host
 * memory: the layer of a serving or inference loop fed from the host.
 *   x_host [n_batches, T, H] bf16 and y_host [n_batches, T, H] fp32 in host memory (page-
 *   locked, e.g. cudaHostAlloc, for the copies to overlap; pageable memory works but the
 *   host then waits for each copy); batch i's layer output is written to y_host[i].
 *   W_gate_up_scale, W_down_scale: NULL for BF16 routed experts (W_gate_up, W_down bf16 as in
 *   moe_forward), or the 128x128 block scales of FP8 E4M3 routed experts (W_gate_up, W_down
 *   the E4M3 codes, as in moe_forward_fp8); both NULL or both given.
 *   Other weights, desc and the routing as in moe_forward; ws of at least
 *   moe_host_workspace_size.
 * The copies run on internal streams, double-buffered in ws: batch i+1's input copy (one
 * stream) and batch i-1's output copy (two halves on two streams) overlap batch i's forward
 * on `stream`. The call only enqueues
 * work; when `stream` has completed, every output row is in y_host. n_batches = 0 or T = 0
 * is a no-op. */
MOE_API moe_status_t moe_forward_host(const moe_layer_desc *desc, int32_t n_batches, const uint16_t *x_host,
                                      const uint16_t *Wr, const float *bias, const void *W_gate_up,
                                      const float *W_gate_up_scale, const void *W_down, const float *W_down_scale,
                                      const uint16_t *Wsh_gate_up, const uint16_t *Wsh_down, float *y_host,
                                      void *ws, size_t ws_bytes, void *stream);

/* ---- Expert parallelism ("MAX 中 Step-3.5-Flash 架构解析", section "并行模式TP_TP / TP_EP /
 * DP_EP": in DP_EP each rank runs its own batch shard, the routed experts are split across
 * ranks and an EP combine follows the MoE; NeMo AutoModel Step-5-Preview page, "Model
 * Architecture" table: expert parallelism, e.g. EP32 with 11 routed experts per rank).
 * With R ranks, rank r owns the routed experts [r*Er, (r+1)*Er), Er = E / R; the router and
 * the shared expert are replicated. One forward on each rank:
 *   moe_router, moe_permute (global E): slots in global expert order = (owner rank, local
 *   expert) order; moe_ep_pack: the send rows; an all-to-all of the per-(owner, local expert)
 *   counts and of the rows (NCCL, by the caller); moe_ep_experts on the received rows; the
 *   reverse all-to-all of their fp32 outputs into rows [0, T*k) of o_perm;
 *   moe_shared_expert into rows [T*k, T*k + T); moe_combine. */

/* Send buffer of a dispatch: x_send[slot_of[t, j]] = x[t], w_send[slot_of[t, j]] = topk_w[t, j]
 * for every routed (token, rank); desc, x [T, H] bf16, topk_w [T, k] fp32 and slot_of [T, k]
 * as in moe_expert_ffn. x_send [T*k, H] bf16 (16-byte aligned), w_send [T*k] fp32. Rows of
 * owner rank r are the slots [offsets[r*Er], offsets[(r+1)*Er]). */
MOE_API moe_status_t moe_ep_pack(const moe_layer_desc *desc, const uint16_t *x, const float *topk_w,
                                 const int32_t *slot_of, uint16_t *x_send, float *w_send, void *stream);

/* Owner side of a dispatch: the routed experts of this rank on the rows it received.
 *   desc: T = rows received, k = 1, E = local experts Er; H, I, Is, limits as the layer
 *         (deterministic is ignored: every output row has one contribution).
 *   ep_ranks R (1..64, R * Er <= 8192); recv_counts [R, Er] int32 on the device: rows that
 *         source rank s sent for local expert e. Rows arrive source-major: all rows of source
 *         0 (its expert 0 rows, then expert 1, ...), then source 1, ...
 *   x_recv [T, H] bf16, w_recv [T] fp32 routing weights of the rows;
 *   W_gate_up [Er, 2I, H], W_down [Er, H, I] bf16: this rank's experts;
 *   out [T, H] fp32 (overwritten): out[n] = w_recv[n] * expert(x_recv[n]), in received order;
 *   ws, ws_bytes: at least moe_workspace_size(desc) bytes.
 * MOE_ERR_INVALID_ARG for k != 1 or R out of range, MOE_ERR_UNSUPPORTED for a count table
 * above 8192 entries. The sum of recv_counts must equal T; rows past the sum are not written. */
MOE_API moe_status_t moe_ep_experts(const moe_layer_desc *desc, int32_t ep_ranks, const int32_t *recv_counts,
                                    const uint16_t *x_recv, const float *w_recv, const uint16_t *W_gate_up,
                                    const uint16_t *W_down, float *out, void *ws, size_t ws_bytes, void *stream);

/* The shared expert alone on this rank's tokens: out[t] = shared_expert(x[t]) with the
 * shared clip limit; x [T, H] bf16, Wsh_gate_up [2Is, H], Wsh_down [H, Is] bf16, out [T, H]
 * fp32 (overwritten; e.g. rows [T*k, T*k + T) of an o_perm for moe_combine); ws of at least
 * moe_workspace_size(desc) bytes. */
MOE_API moe_status_t moe_shared_expert(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wsh_gate_up,
                                       const uint16_t *Wsh_down, float *out, void *ws, size_t ws_bytes,
                                       void *stream);

/* Backward pass of the layer (the layer is trained: NeMo AutoModel Step-5-Preview page,
 * benchmark recipe with forward, backward and optimizer steps; miles page: BF16 training).
 * Given the forward's routing (topk_idx [T,k] int32, topk_w [T,k] fp32, e.g. the outputs of
 * moe_forward) and dy = dLoss/dy [T,H] fp32, overwrites
 *   dx [T,H], dWr [E,H], dW_gate_up [E,2I,H], dW_down [E,H,I], dWsh_gate_up [2Is,H],
 *   dWsh_down [H,Is]   (all fp32, layouts of the corresponding forward tensors).
 * Chain rule on the forward; no gradient flows through the top-k selection (the router
 * bias gets none, so no dbias is produced), clips pass the gradient at their boundary.
 * The router logits of the selected experts are recomputed in fp32. GEMM operands are bf16
 * (dy, the pre-activation gradients and w*h are rounded to bf16), accumulation fp32.
 * Requires I % 128 == 0 and Is % 128 == 0 (MOE_ERR_UNSUPPORTED), every pointer 16-byte
 * aligned; workspace of moe_backward_workspace_size() bytes (about (T*k + 64*E + T) * (4*H
 * + 14*I) bytes). T = 0 returns MOE_OK and writes nothing. */
MOE_API moe_status_t moe_backward_workspace_size(const moe_layer_desc *desc, size_t *bytes);
MOE_API moe_status_t moe_backward(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                                  const uint16_t *W_gate_up, const uint16_t *W_down, const uint16_t *Wsh_gate_up,
                                  const uint16_t *Wsh_down, const int32_t *topk_idx, const float *topk_w,
                                  const float *dy, float *dx, float *dWr, float *dW_gate_up, float *dW_down,
                                  float *dWsh_gate_up, float *dWsh_down, void *ws, size_t ws_bytes, void *stream);

/* moe_forward without a caller-provided workspace. The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory at call time, such
 * as a serving runtime whose device memory is already handed to a fixed pool, a
 * latency-bound decode loop that must avoid cudaMalloc / cudaFree (they can synchronise
 * the device), or a plugin without access to its host framework's allocator.
 * The library keeps one 16 MiB scratch array in device memory and uses it as the
 * workspace; nothing is allocated per call. Under CUDA's default lazy module loading a
 * device gets the array at the first moe_forward_noalloc call made on it (under eager
 * loading, when the library's device code loads), and keeps it until the process exits.
 * Make that first call on each device before any stream capture. Every call looks up the
 * array's device address in the current context (a runtime query, no allocation), so no
 * address outlives its context. Arguments and results are those of moe_forward (inputs
 * and y are still the caller's). A call whose moe_workspace_size() exceeds 16 MiB
 * (16777216 bytes) returns MOE_ERR_WORKSPACE before enqueueing anything; at H = 4096,
 * E = 288, k = 8, I = Is = 1280 the limit is 188 tokens in the default mode and 70 tokens
 * in the deterministic mode (which adds the (T*k + T) x H fp32 per-slot outputs). All
 * calls on a device share the one array: calls whose work overlaps on the GPU (for
 * example on two streams) race and give wrong results; calls on one stream are ordered
 * and safe. Nothing from a previous call needs clearing: every scratch byte read is
 * written first in the same call. */
MOE_API moe_status_t moe_forward_noalloc(const moe_layer_desc *desc, const uint16_t *x, const uint16_t *Wr,
                                 const float *bias, const uint16_t *W_gate_up,
                                 const uint16_t *W_down, const uint16_t *Wsh_gate_up,
                                 const uint16_t *Wsh_down, float *y, int32_t *topk_idx_out,
                                 float *topk_w_out, void *stream);

/* Waits for the current device, then reports and clears the device error word:
 * MOE_ERR_TIMEOUT if a bounded device wait expired since the last call,
 * MOE_ERR_DEVICE_BOUNDS if a range check of the debug build failed, MOE_ERR_CUDA if
 * the device reports an error, else MOE_OK. This call synchronises the device. */
MOE_API moe_status_t moe_check_device(void);

/* Stage timing hook (profiling). When n > 0, every later moe_forward on this process
 * records events[0] before the router, events[1] before the permutation, events[2] before
 * the gather / tile table, events[3] before the gate_up GEMM, events[4] before the down
 * GEMM, events[5] after the down GEMM and, when n >= 7, events[6] after the combine
 * (deterministic mode), each with cudaEventRecord on the call's stream. `events` are
 * cudaEvent_t handles owned by the caller; the array is copied. n = 0 turns it off.
 * Returns MOE_ERR_INVALID_ARG if n < 0, n > 7, or n > 0 and events or one of its
 * entries is NULL. A moe_forward whose event record fails returns MOE_ERR_CUDA. */
MOE_API moe_status_t moe_set_stage_events(void *const *events, int n);

/* Upper bound, in nanoseconds, of every device-side wait in later launches on this
 * process (default 2e9). Values below 1000 are raised to 1000. Returns the old value. */
MOE_API uint64_t moe_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
