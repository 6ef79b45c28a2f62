// epilogue.cuh — TMEM-to-global epilogues of the grouped expert GEMMs (shared by the
// single-CTA, CTA-pair and FP8-weight kernels) and the single-CTA tile decoding.
//
// Layer step ("MAX 中 Step-3.5-Flash 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪"):
// each expert is a SwiGLU MLP with a clipped gated activation; the routed outputs are
// weighted by the routing weights and added to the shared expert's output.
//
// The epilogues run in one epilogue warp that owns TMEM lane quarter q (lanes 32q .. 32q+31) of
// MT accumulators of `bn` fp32 columns each, the accumulators at column offsets m * bn
// from `tmem_tile`; column c of an accumulator is token row row0 + c of the chunk.
#pragma once

#include "gemm_common.cuh"
#include "internal.h"

namespace moe {

// Tile-table header (routed chunks, all chunks); the debug build checks it against the
// table's capacity and clamps a bad header.
__device__ __forceinline__ void table_counts(const int32_t *hdr, int max_chunks, uint32_t *err, int &nrc, int &ntot)
{
    nrc = hdr[0];
    ntot = hdr[1];
    if (!dbg_ok(nrc >= 0 && nrc <= ntot && ntot <= max_chunks, err)) {
        ntot = ntot < 0 ? 0 : (ntot > max_chunks ? max_chunks : ntot);
        nrc = nrc < 0 ? 0 : (nrc > ntot ? ntot : nrc);
    }
}

// Tile-table entry ci = (group, first row, rows, -). The debug build checks it against
// the table's capacity, the row capacities of the routed (rows_r) and shared (rows_s)
// groups and the rows of one tile (cap), and clamps a bad entry into range.
__device__ __forceinline__ int4 chunk_at(const int4 *chunks, int ci, int E, int64_t rows_r, int64_t rows_s,
                                         int max_chunks, int cap, uint32_t *err)
{
    if (!dbg_ok(ci >= 0 && ci < max_chunks, err))
        ci = 0;
    int4 c = chunks[ci];
    if (kDebugChecks) {
        const int64_t span = c.x == E ? rows_s : rows_r;
        const bool ok = c.x >= 0 && c.x <= E && c.z >= 1 && c.z <= cap && c.y >= 0 &&
                        c.y + static_cast<int64_t>(c.z) <= span;
        if (!dbg_ok(ok, err)) {
            c.x = c.x < 0 ? 0 : (c.x > E ? E : c.x);
            const int64_t sp = c.x == E ? rows_s : rows_r;
            c.z = c.z < 1 ? 1 : (c.z > cap ? cap : c.z);
            if (c.z > sp)
                c.z = static_cast<int>(sp);
            if (c.y < 0)
                c.y = 0;
            if (c.y + static_cast<int64_t>(c.z) > sp)
                c.y = static_cast<int>(sp - c.z);
        }
    }
    return c;
}

__device__ __forceinline__ int4 chunk_at(const GateUpArgs &a, int ci)
{
    return chunk_at(a.chunks, ci, a.E, a.rows_r, a.rows_s, a.max_chunks, a.cap, a.err);
}

__device__ __forceinline__ int4 chunk_at(const DownArgs &a, int ci)
{
    return chunk_at(a.chunks, ci, a.E, static_cast<int64_t>(a.T) * a.k, a.T, a.max_chunks, a.cap, a.err);
}

// Destination row of a down-GEMM column (slot rr of group sh ? shared : routed): the token's
// row of y, or the slot's row of o_perm in the deterministic mode. Returns false (and the
// debug build records it) when the row is out of range; the caller skips the column.
__device__ __forceinline__ bool down_dst_row(const DownArgs &a, bool sh, int64_t rr, int64_t &dst_row)
{
    const int64_t shared_base = static_cast<int64_t>(a.T) * a.k;
    if (a.deterministic)
        dst_row = sh ? shared_base + rr : rr;
    else
        dst_row = sh ? rr : a.perm_token[rr];
    return dbg_ok(dst_row >= 0 && dst_row < (a.deterministic ? shared_base + a.T : static_cast<int64_t>(a.T)),
                  a.err);
}

// Tile decoding of the single-CTA grouped GEMMs. gate_up tiles enumerate (routed chunk,
// 64*MT-feature block), then (shared chunk, feature block); down tiles (chunk,
// 128*MT-output-feature block). chunks[ci] = (group, first row, rows).
template <int MT>
__device__ __forceinline__ void decode_gate_up(const GateUpArgs &a, int nrc, int tiles_r, int tile, int &g,
                                               int &row0, int &ntok, int &fb)
{
    int ci;
    if (tile < tiles_r) {
        const int nfb = a.I / (64 * MT);
        ci = tile / nfb;
        fb = tile - ci * nfb;
    } else {
        const int nfb = a.Is / (64 * MT);
        const int tt = tile - tiles_r;
        ci = nrc + tt / nfb;
        fb = tt - (tt / nfb) * nfb;
    }
    const int4 c = chunk_at(a, ci);
    g = c.x;
    row0 = c.y;
    ntok = c.z;
}

template <int MT>
__device__ __forceinline__ void decode_down(const DownArgs &a, int tile, int &g, int &row0, int &ntok, int &fb)
{
    const int nfb = a.H / (128 * MT);
    const int ci = tile / nfb;
    fb = tile - ci * nfb;
    const int4 c = chunk_at(a, ci);
    g = c.x;
    row0 = c.y;
    ntok = c.z;
}

// gate_up: accumulator m holds 64 (gate, up) row pairs interleaved by lane (lane 2i gate
// row i, lane 2i+1 its up row) of features feat0 + 64 m .. feat0 + 64 m + 63. Writes
// h[row0 + c, feature] = act(gate, up) in bf16 for the ntok columns of the chunk, in blocks
// of 32 columns starting at cb0 and cstep apart (several warps may share a lane quarter).
template <int MT>
__device__ __forceinline__ void gate_up_epilogue(uint32_t tmem_tile, int bn, int64_t feat0, int ntok,
                                                 int64_t row0, uint16_t *out, int64_t ld, float L, int q, int lane,
                                                 int cb0 = 0, int cstep = 32)
{
    const int row = q * 32 + lane;
    const int pair = row >> 1;
    const bool is_up = row & 1;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        const int64_t feat = feat0 + m * 64 + pair;
        const uint32_t tb = tmem_tile + m * bn + (static_cast<uint32_t>(q * 32) << 16);
        for (int cb = cb0; cb < ntok; cb += cstep) {
            float v[32];
            tmem_load32(tb + cb, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                // even lane finishes column cb+i (needs the up value), odd lane column
                // cb+16+i (needs the gate value)
                const float send = is_up ? v[i] : v[16 + i];
                const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
                const float gv = is_up ? recv : v[i];
                const float uv = is_up ? v[16 + i] : recv;
                const int col = cb + (is_up ? 16 + i : i);
                const float hv = swiglu_clip(gv, uv, L);
                if (col < ntok)
                    out[(row0 + col) * ld + feat] = __bfloat16_as_ushort(__float2bfloat16_rn(hv));
            }
        }
    }
}

// down: accumulator m holds output features feat0 + 128 m + (lane row). Routed columns
// add w_slot * o into y[token] (fp32 atomics) or store it in o_perm[slot]
// (deterministic mode); shared-expert columns (sh) add o with weight 1.
// Columns are taken in blocks of 32 starting at cb0, cstep apart (several warps may share a
// lane quarter).
template <int MT>
__device__ __forceinline__ void down_epilogue(uint32_t tmem_tile, int bn, int64_t feat0, int ntok, int64_t row0,
                                              bool sh, const DownArgs &a, int q, int lane, int cb0 = 0,
                                              int cstep = 32)
{
    const int64_t f = q * 32 + lane;
    const int64_t H = a.H;
    for (int cb = cb0; cb < ntok; cb += cstep) {
        // lane l fetches the destination row and weight of column cb + l (-1: no column)
        const int mycol = cb + lane;
        int64_t dst_row = -1;
        float wgt = 0.0f;
        if (mycol < ntok) {
            const int64_t rr = row0 + mycol;
            if (!down_dst_row(a, sh, rr, dst_row))
                dst_row = -1;
            wgt = sh ? 1.0f : a.w_perm[rr];
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const int64_t feat = feat0 + m * 128 + f;
            float v[32];
            tmem_load32(tmem_tile + m * bn + (static_cast<uint32_t>(q * 32) << 16) + cb, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int64_t drow = __shfl_sync(0xFFFFFFFFu, dst_row, i);
                const float w = __shfl_sync(0xFFFFFFFFu, wgt, i);
                if (drow >= 0) {
                    float *p = a.out + drow * H + feat;
                    if (a.deterministic)
                        *p = w * v[i];
                    else
                        atomicAdd(p, w * v[i]);
                }
            }
        }
    }
}

}  // namespace moe
