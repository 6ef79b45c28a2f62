// internal.h — launchers shared between the kernel translation units and the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

namespace moe {

// Largest dynamic shared memory a CTA may request on sm_100 (227 KB).
constexpr int kMaxDynSmem = 232448;

struct RouterArgs {
    const float *bias;
    int32_t *idx;
    float *w;
    float *margin;  // may be null
    int T, H, E, k;
    float scale;
    int norm;
    int num_sms;
};
// Router launch geometry: e_pad experts per CTA (E rounded up to 16), ks CTAs per cluster
// splitting K, Wr rows per TMA box (the Wr tensor map must be encoded with this box height).
struct RouterSplit {
    int e_pad, ks, box_rows;
};
RouterSplit router_split(int E, int T, int H, int num_sms);
cudaError_t launch_router(const CUtensorMap &tm_x, const CUtensorMap &tm_wr, const RouterArgs &a,
                          const WaitCfg &wc, cudaStream_t stream);

struct PermuteArgs {
    const int32_t *idx;
    int T, k, E;
    int32_t *counts;      // [E + 1]
    int32_t *offsets;     // [E + 2]
    int32_t *perm_token;  // [T*k + T]
    int32_t *slot_of;     // [T*k]
    const float *topk_w;  // optional, with w_perm: the routing weight of each slot
    float *w_perm;        // [T*k] or null
    int4 *chunks;         // optional tile table of the grouped GEMMs (with hdr, cap)
    int32_t *hdr;
    int cap;
    uint32_t *err;        // device error word (range checks of the debug build)
    int max_chunks;       // capacity of `chunks` (entries)
};
cudaError_t launch_permute(const PermuteArgs &a, cudaStream_t stream);

// Expert-parallel receive side: rows arrive source-major (counts [R, Er] rows per source and
// local expert); writes the expert-major offsets [Er + 2], perm_token and slot_of of the
// received rows. Shared memory of the prefix tables: ep_regroup_smem(R, Er) bytes.
size_t ep_regroup_smem(int R, int Er);
cudaError_t launch_ep_regroup(const int32_t *counts, int R, int Er, int64_t nrows, int32_t *offsets,
                              int32_t *perm_token, int32_t *slot_of, int num_sms, cudaStream_t stream);

// x rows into their routed slots of x_perm (and each slot's routing weight into w_perm); when
// y_zero is not NULL the launch also zeroes its T rows of H fp32 (16-byte aligned). When
// amax_x is not NULL it receives, per routed slot, the largest |x| of the slot's row (float
// bits), and amax_h (same length) is zeroed.
cudaError_t launch_gather(const uint16_t *x, const float *topk_w, const int32_t *slot_of, int T, int k, int H,
                          uint16_t *x_perm, float *w_perm, int num_sms, uint32_t *err, cudaStream_t stream,
                          float *y_zero = nullptr, uint32_t *amax_x = nullptr, uint32_t *amax_h = nullptr);

// Grouped-GEMM configuration. gate_up and down each split every group into chunks of at
// most `cap` / `cap_d` token rows (the N side of one tile) and stage `mt` / `mt_d` 128-row
// weight tiles per pipeline stage and CTA; `pair` = tiles run on CTA pairs (cta_group::2).
// Decode-sized calls (at most 16 tokens per expert on average) use 32-row chunks with one
// weight tile and a deep ring. Larger calls run on CTA pairs when I and Is split into
// 128-feature gate_up pair tiles and H into 512-feature blocks: both GEMMs on chunks of up to
// 256 rows (so most experts of a prefill batch stream their weights once) with one weight
// tile per CTA (gate_up 128 features, down 256 output features per pair tile). Otherwise
// single CTAs take two weight tiles per stage (I, Is multiples of 128, H of 256), else one
// weight tile and 256-row chunks.
constexpr int kPairCapGateUp = 256, kPairMtGateUp = 1, kPairCapDown = 256, kPairMtDown = 1;
// Token rows per TMA box on CTA pairs: the pair kernels get token tensor maps with boxes of
// 32, 64, 96 and 128 rows, and a tile loads one box per K slice, the smallest that covers
// the rows of its CTA half (at most 31 unused rows). Several smaller boxes per slice (16-row
// boxes: up to 18 TMA copies per stage) measured 20-30% slower on gate_up: the single
// producer thread became the bound.
constexpr int kPairTokBoxStep = 32;
constexpr int kPairTokBoxes = 4;  // box heights kPairTokBoxStep * (i + 1)

// Token-row tensor maps of one grouped GEMM: routed rows (x_perm or h) and shared rows (x or
// h_sh) with boxes of the chunk cap on single CTAs, and for the pair kernels the same rows
// with boxes of kPairTokBoxStep * (i + 1) rows (routed_b[i], shared_b[i]).
struct TokMaps {
    CUtensorMap routed, shared;
    CUtensorMap routed_b[kPairTokBoxes], shared_b[kPairTokBoxes];
};
// The pair kernels take their token maps by value in one parameter block.
struct PairTokMaps {
    CUtensorMap routed_b[kPairTokBoxes], shared_b[kPairTokBoxes];
};
struct GemmConfig {
    int cap;
    int mt;
    int cap_d;
    int mt_d;
    int pair;
};
inline GemmConfig gemm_config(int64_t T, int64_t k, int64_t E, int64_t H, int64_t I, int64_t Is)
{
    if (T * k <= 16 * E)
        return {32, 1, 32, 1, 0};
    if (I % 128 == 0 && Is % 128 == 0 && H % 512 == 0)
        return {kPairCapGateUp, kPairMtGateUp, kPairCapDown, kPairMtDown, 1};
    if (I % 128 == 0 && Is % 128 == 0 && H % 256 == 0)
        return {128, 2, 128, 2, 0};
    return {256, 1, 256, 1, 0};
}

// Splits every group (E routed experts, then the shared expert) into chunks of at most
// `cap` rows. hdr[0] = routed chunk count, hdr[1] = total chunk count. When `chunks_d` is
// not NULL the same launch also builds a second table of at most `cap_d` rows per chunk
// (header hdr_d). max_chunks / max_chunks_d: table capacities (range checks of the debug
// build, which also check the offsets against `rows`, the permuted rows' capacity).
cudaError_t launch_chunks(const int32_t *offsets, int E, int T, int cap, int4 *chunks, int32_t *hdr, int cap_d,
                          int4 *chunks_d, int32_t *hdr_d, int max_chunks, int max_chunks_d, int64_t rows,
                          uint32_t *err, cudaStream_t stream);
// FP8-weight configuration (single CTAs, one weight tile per stage): 32-row chunks for
// decode-sized calls, else 128-row chunks.
inline GemmConfig gemm_config_fp8(int64_t T, int64_t k, int64_t E)
{
    if (T * k <= 16 * E)
        return {32, 1, 32, 1, 0};
    return {128, 1, 128, 1, 0};
}

// Upper bound on the chunk count of one table: ceil(n / cap) <= n / cap + 1 per group.
inline int64_t max_chunks(int64_t T, int64_t k, int64_t E, int64_t cap)
{
    return (T * k + T) / cap + E + 2;
}

struct GateUpArgs {
    const int4 *chunks;
    const int32_t *hdr;
    uint16_t *h;     // [T*k, I] bf16
    uint16_t *h_sh;  // [T, Is] bf16
    int E, H, I, Is;
    float lim_r, lim_s;
    const float *w_scale;  // FP8 kernels: block scales [E, 2I/128, H/128]; else unused
    // capacities checked by the debug build: routed rows of x_perm / h, shared rows of
    // h_sh, tile-table entries, rows per tile
    int64_t rows_r, rows_s;
    int max_chunks, cap;
    uint32_t *err;  // device error word
    // FP8 tensor-core kernels: largest |x| of each routed row of x_perm (float bits, read)
    // and of each routed row of h (float bits, raised with atomicMax; zero on entry)
    const uint32_t *amax_in;
    uint32_t *amax_out;
};
cudaError_t launch_gate_up(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const TokMaps &tok,
                           const GateUpArgs &a, const WaitCfg &wc, int grid, const GemmConfig &c,
                           cudaStream_t stream);

struct DownArgs {
    const int4 *chunks;
    const int32_t *hdr;
    const int32_t *perm_token;
    const float *w_perm;
    float *out;  // y [T, H] (atomic) or o_perm [T*k + T, H] (deterministic)
    int E, H, I, Is, T, k;
    int deterministic;
    const float *w_scale;  // FP8 kernels: block scales [E, H/128, I/128]; else unused
    int max_chunks, cap;   // tile-table capacity and rows per tile (debug-build range checks)
    uint32_t *err;         // device error word
    const uint32_t *amax_in;  // FP8 tensor-core kernels: largest |h| of each routed row (float bits)
};
cudaError_t launch_down(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const TokMaps &tok,
                        const DownArgs &a, const WaitCfg &wc, int grid, const GemmConfig &c, cudaStream_t stream);

cudaError_t launch_gate_up_pair(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const TokMaps &tok,
                                const GateUpArgs &a, const WaitCfg &wc, int grid, cudaStream_t stream);
cudaError_t launch_down_pair(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const TokMaps &tok,
                             const DownArgs &a, const WaitCfg &wc, int grid, cudaStream_t stream);

// FP8 E4M3 routed experts (128x128 block scales, shared expert BF16): tm_w / tm_wd map
// the E4M3 codes (gate_up: 4-D (H, half, row, expert) bytes; down: 2-D (I, E*H) bytes).
cudaError_t launch_gate_up_fp8(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const CUtensorMap &tm_xp,
                               const CUtensorMap &tm_x, const GateUpArgs &a, const WaitCfg &wc, int grid,
                               const GemmConfig &c, cudaStream_t stream);
cudaError_t launch_down_fp8(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const CUtensorMap &tm_h,
                            const CUtensorMap &tm_hsh, const DownArgs &a, const WaitCfg &wc, int grid,
                            const GemmConfig &c, cudaStream_t stream);

// FP8 E4M3 routed experts on the FP8 tensor cores (tcgen05 kind::f8f6f4), decode-sized
// calls: tiles of two 128-row weight blocks (gate_up: 128 gate rows and their up rows; down:
// 256 output rows), 32-row chunks, the block scales applied to the token operand. Needs H a
// multiple of 256 and I, Is multiples of 128. tm_w / tm_wd: the E4M3 codes as 2-D (H, E*2I)
// / (I, E*H) bytes with 128 x 128 boxes; tm_wsh / tm_wdsh: the BF16 shared expert as (H, 2Is)
// / (Is, H) with 64 x 128 boxes; token maps with 32-row boxes. GateUpArgs::amax_in /
// amax_out and DownArgs::amax_in must be set.
inline bool fp8_mma_config(const GemmConfig &c, int64_t H, int64_t I, int64_t Is)
{
    return c.cap == 32 && c.cap_d == 32 && H % 256 == 0 && I % 128 == 0 && Is % 128 == 0;
}
cudaError_t launch_gate_up_fp8_mma(const CUtensorMap &tm_w, const CUtensorMap &tm_wsh, const CUtensorMap &tm_xp,
                                   const CUtensorMap &tm_x, const GateUpArgs &a, const WaitCfg &wc, int grid,
                                   cudaStream_t stream);
cudaError_t launch_down_fp8_mma(const CUtensorMap &tm_wd, const CUtensorMap &tm_wdsh, const CUtensorMap &tm_h,
                                const CUtensorMap &tm_hsh, const DownArgs &a, const WaitCfg &wc, int grid,
                                cudaStream_t stream);

// ------------------------------------------------------------------------------------
// Backward pass. Rows live in a padded permuted space: the shared group takes rows [0, T)
// of a span of P_s = T rounded up to 64 rows, then routed group e occupies rows
// [poff[e], poff[e] + count[e]) of a span rounded up to 64 rows; padding rows are zero in
// x_pad / dy_pad, so the weight-gradient GEMMs reduce over whole 64-row K slices. chunks: tiles of <= kBwdCap valid rows (group, first
// row, rows); wgroups: (group, first row, padded rows). hdr: [0] routed chunks, [1] all
// chunks, [2] routed wgroups, [3] all wgroups.
constexpr int kBwdCap = 256;
constexpr int kBwdPad = 64;
struct BwdArgs {
    int T, H, E, k, I, Is;
    float lim_r, lim_s;
    int P_s;  // rows of the shared group's span = first routed row
    const int4 *chunks;
    const int4 *wgroups;
    const int32_t *hdr;
    const float *w_pad;      // [P] routing weight of the row (1 for shared rows, 0 for padding)
    const int32_t *tok_pad;  // [P] token of the row (-1 for padding)
    float *gu_r, *gu_s;      // pre-activations [rows - P_s, 2I] / [P_s, 2Is] fp32 (gate columns, then up)
    uint16_t *dgu_r, *dgu_s;  // gradients of the pre-activations, same shapes, bf16
    uint16_t *hw_r, *hw_s;    // w * h [rows - P_s, I] / [P_s, Is] bf16
    float *dw_pad;            // [P] dLoss/dw of routed rows (accumulated)
    float *dx;                // [T, H]
    float *dWd, *dWgu, *dWsh_d, *dWsh_gu;
    const int32_t *counts;    // [E] rows per routed expert (DH zeroes the gradients of those with none)
};
enum BwdMode { kBwdGU = 0, kBwdDH = 1, kBwdDX = 2, kBwdWD = 3, kBwdWGU = 4 };
// Maps per mode (routed A, shared A, routed B, shared B):
//   GU : W_gate_up / Wsh_gate_up (4-D gate/up interleave, K-major), x_pad, x_pad
//   DH : W_down / Wsh_down as (I, rows) MN-major, dy_pad, dy_pad
//   DX : W_gate_up / Wsh_gate_up as (H, rows) MN-major, dgu_r, dgu_s (K-major)
//   WD : dy_pad (H, rows) MN-major (both), hw_r / hw_s (I, rows) MN-major
//   WGU: dgu_r / dgu_s (2I, rows) MN-major, x_pad (H, rows) MN-major (both)
// and, last, two more maps (routed, shared): for the weight-gradient modes their fp32 outputs,
// 32 x 32 boxes with 128-byte swizzle (WD dW_down (I, E*H) / dWsh_down (Is, H), WGU
// dW_gate_up (H, E*2I) / dWsh_gate_up (H, 2Is)); for GU, DH and DX the same token rows as
// their B maps with 128-row boxes (the B maps have kBwdCap-row boxes; a chunk of at most 128
// rows loads the smaller box).
cudaError_t launch_bwd_gemm(int mode, const CUtensorMap &a_r, const CUtensorMap &a_s, const CUtensorMap &b_r,
                            const CUtensorMap &b_s, const CUtensorMap &o_r, const CUtensorMap &o_s, const BwdArgs &a,
                            const WaitCfg &wc, int grid, cudaStream_t stream);
// Padded layout + tile tables from the permutation's counts (one CTA).
cudaError_t launch_bwd_layout(const int32_t *counts, int E, int T, int32_t *poff, int4 *chunks, int4 *wgroups,
                              int32_t *hdr, cudaStream_t stream);
// x_pad, dy_pad (bf16 of dy), w_pad, tok_pad from the forward's routing; padding rows zero.
cudaError_t launch_bwd_gather(const uint16_t *x, const float *dy, const int32_t *topk_idx, const float *topk_w,
                              const int32_t *slot_of, const int32_t *offsets, const int32_t *counts,
                              const int32_t *poff, int T, int k, int E, int H, uint16_t *x_pad, uint16_t *dy_pad,
                              float *w_pad, int32_t *tok_pad, cudaStream_t stream);
// Router part: logits of the selected experts, dLoss/dlogit, dx = sum_j dlogit_j Wr[e_j]
// (overwrites dx) and dlogit per padded row (dl_pad).
cudaError_t launch_bwd_router(const uint16_t *x, const uint16_t *Wr, const int32_t *topk_idx, const int32_t *slot_of,
                              const int32_t *offsets, const int32_t *poff, const float *dw_pad, int T, int k, int E,
                              int H, float scale, int norm, float *dx, float *dl_pad, cudaStream_t stream);
// dWr[e] = sum of dl_pad[row] * x_pad[row] over group e's rows.
cudaError_t launch_bwd_dwr(const uint16_t *x_pad, const float *dl_pad, const int32_t *poff, const int32_t *counts,
                           int E, int H, float *dWr, cudaStream_t stream);

cudaError_t launch_combine(const float *o_perm, const int32_t *slot_of, int T, int k, int H, float *y,
                           uint32_t *err, cudaStream_t stream);

}  // namespace moe
