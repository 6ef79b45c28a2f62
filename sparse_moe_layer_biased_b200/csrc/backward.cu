// backward.cu — backward pass of the MoE FFN layer on sm_100a.
//
// The layer is trained (NeMo AutoModel Step-5-Preview page, benchmark recipe: forward,
// backward and optimizer steps; miles Step-5-Preview page: BF16 training). The pages give
// no formulas; the gradients are the chain rule on the forward ("MAX 中 Step-3.5-Flash
// 架构解析", section "MoE共享专家、sigmoid 路由与激活裁剪"), with no gradient through the top-k
// selection (the router bias gets none) and clips that pass the gradient at their boundary.
//
// Given the forward's routing (ids, weights) and dy = dLoss/dy:
//   GU   pre-activations g, u of every (token, expert) row recomputed: x_pad · W_gate_upᵀ
//   DH   dhu = dy_pad · W_down (A = W_downᵀ read MN-major); epilogue: dw = h · dhu,
//        dh = w dhu, dg = dh u_c silu'(g) [a <= L], du = dh a_c [|u| <= L]
//   router  s of the selected experts recomputed, dlogit = ds s (1 - s), dx = Σ dlogit Wr[e]
//   DX   dx += W_gate_upᵀ · [dg du] (A = W_gate_upᵀ read MN-major), scattered to tokens
//   WD   dW_down_e = Σ_rows dy_padᵀ (w h)   (both operands MN-major, K = the group's rows)
//   WGU  dW_gate_up_e = Σ_rows [dg du]ᵀ x_pad
//   dWr  dWr[e] = Σ_rows dlogit x_pad
// Rows live in a padded permuted space (each group rounded up to 64 rows, padding zero) so
// the weight-gradient GEMMs reduce over whole 64-row K slices.
#include "epilogue.cuh"

namespace moe {
namespace {

constexpr int kLayoutThreads = 1024;

// Exclusive block-wide prefix sum of v over the 1024 threads; returns the total in *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_sums, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o)
            incl += t;
    }
    if (lane == 31)
        warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int ws = warp_sums[lane];
        int wi = ws;
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o)
                wi += t;
        }
        warp_sums[lane] = wi - ws;
        if (lane == 31)
            *total = wi;
    }
    __syncthreads();
    const int r = warp_sums[warp] + incl - v;
    __syncthreads();
    return r;
}

// One CTA: padded group offsets poff[0..E+1], the chunk table (rows of a group split into
// ceil(n / cap) near-equal chunks, rounded to 16 rows) and the weight-gradient group table.
__global__ void __launch_bounds__(kLayoutThreads)
    bwd_layout_kernel(const int32_t *__restrict__ counts, int E, int T, int32_t *__restrict__ poff,
                      int4 *__restrict__ chunks, int4 *__restrict__ wgroups, int32_t *__restrict__ hdr)
{
    __shared__ int warp_sums[32];
    __shared__ int totals[3];
    const int g = threadIdx.x;  // E + 1 <= 513 < 1024 groups: one pass
    int n = 0;
    if (g < E)
        n = counts[g];
    else if (g == E)
        n = T;
    const int padded = (n + kBwdPad - 1) / kBwdPad * kBwdPad;
    const int nch = n > 0 ? (n + kBwdCap - 1) / kBwdCap : 0;
    const int nwg = n > 0 ? 1 : 0;
    // the shared group (g = E) comes first in rows, the routed groups after it
    const int P_s = (T + kBwdPad - 1) / kBwdPad * kBwdPad;
    const int pre = block_exclusive_scan(g < E ? padded : 0, warp_sums, &totals[0]);  // every thread scans
    const int row0 = g == E ? 0 : P_s + pre;
    const int c0 = block_exclusive_scan(nch, warp_sums, &totals[1]);
    const int w0 = block_exclusive_scan(nwg, warp_sums, &totals[2]);
    if (g <= E) {
        poff[g] = row0;
        const int csz = nch > 0 ? ((n + nch - 1) / nch + 15) / 16 * 16 : 0;
        for (int c = 0; c < nch; ++c) {
            const int r = c * csz;
            chunks[c0 + c] = make_int4(g, row0 + r, n - r < csz ? n - r : csz, 0);
        }
        if (nwg)
            wgroups[w0] = make_int4(g, row0, padded, 0);
        if (g == E) {
            poff[E + 1] = P_s + totals[0];
            hdr[0] = c0;
            hdr[1] = c0 + nch;
            hdr[2] = w0;
            hdr[3] = w0 + nwg;
        }
    }
}

// One warp per (token, rank) pair (and per token for the shared group): copies x[t] and
// bf16(dy[t]) into the pair's padded row; extra blocks zero the padding rows.
__global__ void __launch_bounds__(256)
    bwd_gather_kernel(const uint16_t *__restrict__ x, const float *__restrict__ dy, const int32_t *__restrict__ idx,
                      const float *__restrict__ topk_w, const int32_t *__restrict__ slot_of,
                      const int32_t *__restrict__ offsets, const int32_t *__restrict__ counts,
                      const int32_t *__restrict__ poff, int T, int k, int E, int H, uint16_t *__restrict__ x_pad,
                      uint16_t *__restrict__ dy_pad, float *__restrict__ w_pad, int32_t *__restrict__ tok_pad,
                      int pair_blocks)
{
    const int lane = threadIdx.x & 31;
    if (static_cast<int>(blockIdx.x) >= pair_blocks) {
        // padding rows of group g = blockIdx.x - pair_blocks
        // group spans: shared [0, P_s), routed e [poff[e], poff[e + 1]), the last routed one
        // ending at poff[E + 1]
        const int g = blockIdx.x - pair_blocks;
        const int n = g < E ? counts[g] : T;
        const int64_t r0 = poff[g] + n;
        const int64_t r1 = g == E ? (T + kBwdPad - 1) / kBwdPad * kBwdPad : (g + 1 < E ? poff[g + 1] : poff[E + 1]);
        for (int64_t r = r0 + (threadIdx.x >> 5); r < r1; r += 8) {
            for (int h = lane * 8; h < H; h += 256) {
                *reinterpret_cast<uint4 *>(x_pad + r * H + h) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(dy_pad + r * H + h) = make_uint4(0, 0, 0, 0);
            }
            if (lane == 0) {
                w_pad[r] = 0.0f;
                tok_pad[r] = -1;
            }
        }
        return;
    }
    const int64_t pairs = static_cast<int64_t>(T) * k + T;
    for (int64_t n = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); n < pairs;
         n += static_cast<int64_t>(pair_blocks) * 8) {
        int64_t t, row;
        float w;
        if (n < static_cast<int64_t>(T) * k) {
            t = n / k;
            int e = idx[n];
            e = e < 0 ? 0 : (e > E - 1 ? E - 1 : e);
            row = poff[e] + (slot_of[n] - offsets[e]);
            w = topk_w[n];
        } else {
            t = n - static_cast<int64_t>(T) * k;
            row = poff[E] + t;
            w = 1.0f;
        }
        for (int h = lane * 8; h < H; h += 256) {
            *reinterpret_cast<uint4 *>(x_pad + row * H + h) = *reinterpret_cast<const uint4 *>(x + t * H + h);
            const float4 a = *reinterpret_cast<const float4 *>(dy + t * H + h);
            const float4 b = *reinterpret_cast<const float4 *>(dy + t * H + h + 4);
            __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
            __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
            uint4 o;
            o.x = *reinterpret_cast<uint32_t *>(&p0);
            o.y = *reinterpret_cast<uint32_t *>(&p1);
            o.z = *reinterpret_cast<uint32_t *>(&p2);
            o.w = *reinterpret_cast<uint32_t *>(&p3);
            *reinterpret_cast<uint4 *>(dy_pad + row * H + h) = o;
        }
        if (lane == 0) {
            w_pad[row] = w;
            tok_pad[row] = static_cast<int32_t>(t);
        }
    }
}

// One warp per token: logits of its k selected experts (fp32 dot products), scores,
// dLoss/ds through the normalised scaled weights, dLoss/dlogit = ds s (1 - s);
// dx[t] = Σ_j dlogit_j Wr[e_j] (overwrites dx) and dl_pad[row of (t, j)] = dlogit_j.
__global__ void __launch_bounds__(256)
    bwd_router_kernel(const uint16_t *__restrict__ x, const uint16_t *__restrict__ Wr, const int32_t *__restrict__ idx,
                      const int32_t *__restrict__ slot_of, const int32_t *__restrict__ offsets,
                      const int32_t *__restrict__ poff, const float *__restrict__ dw_pad, int T, int k, int E, int H,
                      float scale, int norm, float *__restrict__ dx, float *__restrict__ dl_pad)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (t >= T)
        return;
    float s[32], dw[32];
    int ex[32];
    int64_t rows[32];
    float Z = 0.0f, sdw = 0.0f;
    for (int j = 0; j < k; ++j) {
        int e = idx[t * k + j];
        e = e < 0 ? 0 : (e > E - 1 ? E - 1 : e);
        const uint16_t *wr = Wr + static_cast<int64_t>(e) * H;
        const uint16_t *xr = x + t * H;
        float acc = 0.0f;
        for (int h = lane * 2; h < H; h += 64) {
            const __nv_bfloat162 xv = *reinterpret_cast<const __nv_bfloat162 *>(xr + h);
            const __nv_bfloat162 wv = *reinterpret_cast<const __nv_bfloat162 *>(wr + h);
            const float2 xf = __bfloat1622float2(xv), wf = __bfloat1622float2(wv);
            acc = fmaf(xf.x, wf.x, acc);
            acc = fmaf(xf.y, wf.y, acc);
        }
        for (int o = 16; o > 0; o >>= 1)
            acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        const float sj = 1.0f / (1.0f + expf(-acc));
        const int64_t row = poff[e] + (slot_of[t * k + j] - offsets[e]);
        const float dwj = dw_pad[row];
        s[j] = sj;
        dw[j] = dwj;
        ex[j] = e;
        rows[j] = row;
        Z += sj;
        sdw += dwj * sj;
    }
    for (int j = 0; j < k; ++j) {
        float ds;
        if (!norm)
            ds = scale * dw[j];
        else if (Z > 0.0f)
            ds = scale / Z * dw[j] - scale / (Z * Z) * sdw;
        else
            ds = 0.0f;  // all selected scores underflowed: the weights are the constant scale/k
        s[j] = ds * s[j] * (1.0f - s[j]);  // dlogit
        if (lane == 0)
            dl_pad[rows[j]] = s[j];
    }
    for (int h = lane * 2; h < H; h += 64) {
        float a0 = 0.0f, a1 = 0.0f;
        for (int j = 0; j < k; ++j) {
            const float2 wf =
                __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(Wr + static_cast<int64_t>(ex[j]) * H + h));
            a0 = fmaf(s[j], wf.x, a0);
            a1 = fmaf(s[j], wf.y, a1);
        }
        *reinterpret_cast<float2 *>(dx + t * H + h) = make_float2(a0, a1);
    }
}

// dWr[e][h] = Σ over group e's rows of dl_pad[row] * x_pad[row][h]. Block (e, 512 columns,
// split z of kDwrSplit) sums rows r0 + z, r0 + z + kDwrSplit, ... (four rows of loads in flight)
// and adds its partial sums into dWr, which the launch zeroes first: a hot expert's thousands
// of rows no longer run as one block's serial loop.
constexpr int kDwrSplit = 8;

__global__ void __launch_bounds__(256)
    bwd_dwr_kernel(const uint16_t *__restrict__ x_pad, const float *__restrict__ dl_pad,
                   const int32_t *__restrict__ poff, const int32_t *__restrict__ counts, int E, int H,
                   float *__restrict__ dWr)
{
    const int e = blockIdx.x;
    const int h = blockIdx.y * 512 + threadIdx.x * 2;
    const int64_t r0 = poff[e], r1 = r0 + counts[e];
    if (h >= H || r0 + blockIdx.z >= r1)
        return;
    float a0 = 0.0f, a1 = 0.0f;
    const int64_t step = kDwrSplit;
    int64_t r = r0 + blockIdx.z;
    for (; r + 3 * step < r1; r += 4 * step) {
        float d[4];
        float2 xf[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            d[u] = dl_pad[r + u * step];
            xf[u] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(x_pad + (r + u * step) * H + h));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            a0 = fmaf(d[u], xf[u].x, a0);
            a1 = fmaf(d[u], xf[u].y, a1);
        }
    }
    for (; r < r1; r += step) {
        const float d = dl_pad[r];
        const float2 xf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(x_pad + r * H + h));
        a0 = fmaf(d, xf.x, a0);
        a1 = fmaf(d, xf.y, a1);
    }
    float *out = dWr + static_cast<int64_t>(e) * H + h;
    atomicAdd(out, a0);
    atomicAdd(out + 1, a1);
}

}  // namespace

cudaError_t launch_bwd_layout(const int32_t *counts, int E, int T, int32_t *poff, int4 *chunks, int4 *wgroups,
                              int32_t *hdr, cudaStream_t stream)
{
    bwd_layout_kernel<<<1, kLayoutThreads, 0, stream>>>(counts, E, T, poff, chunks, wgroups, hdr);
    return cudaGetLastError();
}

cudaError_t launch_bwd_gather(const uint16_t *x, const float *dy, const int32_t *topk_idx, const float *topk_w,
                              const int32_t *slot_of, const int32_t *offsets, const int32_t *counts,
                              const int32_t *poff, int T, int k, int E, int H, uint16_t *x_pad, uint16_t *dy_pad,
                              float *w_pad, int32_t *tok_pad, cudaStream_t stream)
{
    const int64_t pairs = static_cast<int64_t>(T) * k + T;
    const int pair_blocks = static_cast<int>((pairs + 7) / 8 < 65536 ? (pairs + 7) / 8 : 65536);
    bwd_gather_kernel<<<pair_blocks + E + 1, 256, 0, stream>>>(x, dy, topk_idx, topk_w, slot_of, offsets, counts,
                                                               poff, T, k, E, H, x_pad, dy_pad, w_pad, tok_pad,
                                                               pair_blocks);
    return cudaGetLastError();
}

cudaError_t launch_bwd_router(const uint16_t *x, const uint16_t *Wr, const int32_t *topk_idx, const int32_t *slot_of,
                              const int32_t *offsets, const int32_t *poff, const float *dw_pad, int T, int k, int E,
                              int H, float scale, int norm, float *dx, float *dl_pad, cudaStream_t stream)
{
    bwd_router_kernel<<<(T + 7) / 8, 256, 0, stream>>>(x, Wr, topk_idx, slot_of, offsets, poff, dw_pad, T, k, E, H,
                                                       scale, norm, dx, dl_pad);
    return cudaGetLastError();
}

cudaError_t launch_bwd_dwr(const uint16_t *x_pad, const float *dl_pad, const int32_t *poff, const int32_t *counts,
                           int E, int H, float *dWr, cudaStream_t stream)
{
    cudaError_t err = cudaMemsetAsync(dWr, 0, static_cast<size_t>(E) * H * 4, stream);
    if (err != cudaSuccess)
        return err;
    bwd_dwr_kernel<<<dim3(E, (H + 511) / 512, kDwrSplit), 256, 0, stream>>>(x_pad, dl_pad, poff, counts, E, H, dWr);
    return cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Grouped GEMMs of the backward pass. One persistent kernel per mode, one CTA per SM, 192
// threads (warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 2..5 epilogue).
// A tile is 128 rows of the output's M side x N columns: up to kBwdCap = 256 token rows in the
// row-streaming modes (GU, DH, DX), kBwdBN = 128 output columns in the weight-gradient modes
// (WD, WGU). A pipeline stage holds one 64-wide K slice of A (16 KB) and B (32 KB of token rows,
// or 16 KB MN-major); a chunk of at most 128 rows loads a 128-row token box. A and B are
// K-major (128-byte rows of K) or MN-major (two 8 KB chunks of 64 MN elements x 64 K rows), as
// the mode's global layout gives them; two TMEM accumulators of 256 columns let the epilogue
// of one tile overlap the next tile's mainloop. 256-row tiles halve the bytes each MMA column
// needs from L2 against 128-row ones (each weight tile streams once per 256 rows).
namespace {

constexpr int kBwdThreads = 192;
// The DH kernel has eight epilogue warps (its per-element SwiGLU derivative work is the
// longest epilogue; the two warps of a lane quarter take alternate 16-column blocks) and one
// more warp that zeroes the weight gradients of routed experts that received no tokens (no
// weight-gradient tile writes them) while the GEMM streams W_down.
constexpr int kBwdDhHalves = 2;
constexpr int kBwdDhEpiWarps = 4 * kBwdDhHalves;
constexpr int kBwdThreadsDH = 32 * (2 + kBwdDhEpiWarps + 1);
constexpr uint32_t kBwdZeroBytes = 2048;  // zero source of those bulk stores
constexpr int kBwdStages = 6;  // stages of 32 KB (the ring region's size in those units)
constexpr int kBwdBN = 128;    // output columns of a weight-gradient tile
constexpr int kBwdAcc = kBwdCap;  // TMEM columns of one accumulator buffer
constexpr uint32_t kBwdTile = 16384;  // A operand (or MN-major B) per K slice
constexpr uint32_t kBwdStage = 2 * kBwdTile;
constexpr uint32_t kBwdBarOff = kBwdStages * kBwdStage;
constexpr uint32_t kBwdMiscOff = kBwdBarOff + 8 * (2 * kBwdStages + 5);
// per epilogue warp: two 4 KB staging boxes of the weight-gradient stores (1024-byte aligned
// for the 128-byte swizzle), or the DH mode's 32 x 33 fp32 transpose
constexpr uint32_t kBwdEpiOff = (kBwdMiscOff + 16 + 1023) / 1024 * 1024;
constexpr uint32_t kBwdEpiBox = 32 * 32 * 4;
constexpr uint32_t kBwdEpiWarp = 2 * kBwdEpiBox;
// DH: a 32 x 17 fp32 transpose buffer per epilogue warp, and the zero source at the end of
// the epilogue area
constexpr uint32_t kBwdDhTr = 2304;
constexpr uint32_t kBwdZeroOff = kBwdEpiOff + 4 * kBwdEpiWarp - kBwdZeroBytes;
static_assert(32 * 17 * 4 <= kBwdDhTr, "transpose buffer");
static_assert(kBwdDhEpiWarps * kBwdDhTr <= 4 * kBwdEpiWarp - kBwdZeroBytes, "zero source overlaps the transpose buffers");
constexpr uint32_t kBwdSmem = kBwdEpiOff + 4 * kBwdEpiWarp + 1024;
static_assert(kBwdSmem <= kMaxDynSmem, "backward ring exceeds shared memory");

// MN-major operand in 128-byte swizzle: 64-element MN chunks lbo bytes apart, 8-row K
// groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo)
{
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
    d |= static_cast<uint64_t>(1024 >> 4) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

struct BTile {
    int g, row0, ntok, mb, nb, K;
    bool sh;
};

template <int MODE>
__device__ __forceinline__ int bwd_tile_count(const BwdArgs &a)
{
    if (MODE == kBwdWD || MODE == kBwdWGU) {
        const int r = a.hdr[2], all = a.hdr[3];
        const int per_r = MODE == kBwdWD ? (a.H / 128) * (a.I / kBwdBN) : (2 * a.I / 128) * (a.H / kBwdBN);
        const int per_s = MODE == kBwdWD ? (a.H / 128) * (a.Is / kBwdBN) : (2 * a.Is / 128) * (a.H / kBwdBN);
        return r * per_r + (all - r) * per_s;
    }
    const int r = a.hdr[0], all = a.hdr[1];
    const int per_r = MODE == kBwdGU ? a.I / 64 : (MODE == kBwdDH ? a.I / 128 : a.H / 128);
    const int per_s = MODE == kBwdGU ? a.Is / 64 : (MODE == kBwdDH ? a.Is / 128 : a.H / 128);
    return r * per_r + (all - r) * per_s;
}

template <int MODE>
__device__ __forceinline__ BTile bwd_tile(const BwdArgs &a, int tile)
{
    BTile t;
    if (MODE == kBwdWD || MODE == kBwdWGU) {
        const int r = a.hdr[2];
        const int nm_r = MODE == kBwdWD ? a.H / 128 : 2 * a.I / 128;
        const int nn_r = MODE == kBwdWD ? a.I / kBwdBN : a.H / kBwdBN;
        const int nm_s = MODE == kBwdWD ? a.H / 128 : 2 * a.Is / 128;
        const int nn_s = MODE == kBwdWD ? a.Is / kBwdBN : a.H / kBwdBN;
        int gi, rem, nn;
        if (tile < r * nm_r * nn_r) {
            gi = tile / (nm_r * nn_r);
            rem = tile - gi * nm_r * nn_r;
            nn = nn_r;
        } else {
            const int tt = tile - r * nm_r * nn_r;
            gi = r + tt / (nm_s * nn_s);
            rem = tt - (tt / (nm_s * nn_s)) * nm_s * nn_s;
            nn = nn_s;
        }
        const int4 w = a.wgroups[gi];
        t.g = w.x;
        t.row0 = w.y;
        t.K = w.z;
        t.ntok = kBwdBN;
        t.mb = rem / nn;
        t.nb = rem - t.mb * nn;
        t.sh = t.g == a.E;
        return t;
    }
    const int r = a.hdr[0];
    const int nm_r = MODE == kBwdGU ? a.I / 64 : (MODE == kBwdDH ? a.I / 128 : a.H / 128);
    const int nm_s = MODE == kBwdGU ? a.Is / 64 : (MODE == kBwdDH ? a.Is / 128 : a.H / 128);
    int ci;
    if (tile < r * nm_r) {
        ci = tile / nm_r;
        t.mb = tile - ci * nm_r;
    } else {
        const int tt = tile - r * nm_r;
        ci = r + tt / nm_s;
        t.mb = tt - (tt / nm_s) * nm_s;
    }
    const int4 c = a.chunks[ci];
    t.g = c.x;
    t.row0 = c.y;
    t.ntok = c.z;
    t.nb = 0;
    t.sh = t.g == a.E;
    const int Iw = t.sh ? a.Is : a.I;
    t.K = MODE == kBwdDX ? 2 * Iw : a.H;
    return t;
}

// Loads of K slice k0 of tile t: A (128 M rows) and B (128 N rows) into a stage.
template <int MODE>
__device__ __forceinline__ void bwd_load(const BwdArgs &a, const CUtensorMap *ma, const CUtensorMap *mb,
                                         uint8_t *A, uint8_t *B, uint64_t *bar, const BTile &t, int k0)
{
    const int Iw = t.sh ? a.Is : a.I;
    const int rs = t.sh ? t.row0 : t.row0 - a.P_s;  // row in the group-split buffers (gu, dgu, hw)
    if (MODE == kBwdGU) {
        tma_load_4d(A, ma, bar, k0, 0, t.mb * 64, t.sh ? 0 : t.g);
        tma_load_2d(B, mb, bar, k0, t.row0);
    } else if (MODE == kBwdDH) {
        const int wrow = (t.sh ? 0 : t.g * a.H) + k0;  // B: mb is the map of the tile's box height
        tma_load_2d(A, ma, bar, t.mb * 128, wrow);
        tma_load_2d(A + 8192, ma, bar, t.mb * 128 + 64, wrow);
        tma_load_2d(B, mb, bar, k0, t.row0);
    } else if (MODE == kBwdDX) {
        const int wrow = (t.sh ? 0 : t.g * 2 * Iw) + k0;
        tma_load_2d(A, ma, bar, t.mb * 128, wrow);
        tma_load_2d(A + 8192, ma, bar, t.mb * 128 + 64, wrow);
        tma_load_2d(B, mb, bar, k0, rs);
    } else if (MODE == kBwdWD) {
        tma_load_2d(A, ma, bar, t.mb * 128, t.row0 + k0);
        tma_load_2d(A + 8192, ma, bar, t.mb * 128 + 64, t.row0 + k0);
        tma_load_2d(B, mb, bar, t.nb * kBwdBN, rs + k0);
        tma_load_2d(B + 8192, mb, bar, t.nb * kBwdBN + 64, rs + k0);
    } else {
        tma_load_2d(A, ma, bar, t.mb * 128, rs + k0);
        tma_load_2d(A + 8192, ma, bar, t.mb * 128 + 64, rs + k0);
        tma_load_2d(B, mb, bar, t.nb * kBwdBN, t.row0 + k0);
        tma_load_2d(B + 8192, mb, bar, t.nb * kBwdBN + 64, t.row0 + k0);
    }
}

// Epilogue of one tile for one warp (TMEM lane quarter q; lane row = q*32 + lane of M; in DH
// the warp's half of the column blocks). om = tensor map of the tile's weight-gradient output (WD / WGU), 32 x 32 fp32 boxes with
// 128-byte swizzle; tr = this warp's staging area (kBwdEpiWarp bytes, 1024-byte aligned).
template <int MODE>
__device__ __forceinline__ void bwd_epilogue(const BwdArgs &a, uint32_t tacc, const BTile &t, int q, int half,
                                             int lane, float *tr, const CUtensorMap *om)
{
    const int row = q * 32 + lane;
    const uint32_t tq = tacc + (static_cast<uint32_t>(q * 32) << 16);
    const int Iw = t.sh ? a.Is : a.I;
    const int64_t rs = t.sh ? t.row0 : t.row0 - a.P_s;
    if (MODE == kBwdGU) {
        // rows interleave gate row f / up row f (lanes 2i, 2i+1) of features mb*64 + i
        const int64_t f = t.mb * 64 + (row >> 1);
        const bool is_up = row & 1;
        float *gu = t.sh ? a.gu_s : a.gu_r;
        uint16_t *hw = t.sh ? a.hw_s : a.hw_r;
        const float L = t.sh ? a.lim_s : a.lim_r;
        for (int cb = 0; cb < t.ntok; cb += 32) {
            float v[32];
            tmem_load32(tq + cb, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (cb + i < t.ntok)
                    gu[(rs + cb + i) * 2 * Iw + f + (is_up ? Iw : 0)] = v[i];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float send = is_up ? v[i] : v[16 + i];
                const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 1);
                const float gv = is_up ? recv : v[i];
                const float uv = is_up ? v[16 + i] : recv;
                const int col = cb + (is_up ? 16 + i : i);
                if (col < t.ntok) {
                    const float w = t.sh ? 1.0f : a.w_pad[t.row0 + col];
                    hw[(rs + col) * Iw + f] = __bfloat16_as_ushort(__float2bfloat16_rn(w * swiglu_clip(gv, uv, L)));
                }
            }
        }
    } else if (MODE == kBwdDH) {
        // blocks of 16 columns; the two warps of a lane quarter take alternate blocks
        const int64_t i = t.mb * 128 + row;
        const float *gu = t.sh ? a.gu_s : a.gu_r;
        uint16_t *dgu = t.sh ? a.dgu_s : a.dgu_r;
        const float L = t.sh ? a.lim_s : a.lim_r;
        for (int cb = 16 * half; cb < t.ntok; cb += 16 * kBwdDhHalves) {
            float v[16], gg[16], uu[16];
            tmem_load16(tq + cb, v);
            const int ncol = t.ntok - cb < 16 ? t.ntok - cb : 16;
            // lane c < 16: routing weight of column cb + c (read by shuffle below)
            const float wl = t.sh || lane >= ncol ? 1.0f : a.w_pad[t.row0 + cb + lane];
            // all 32 pre-activation loads of the block in flight before any use
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const int64_t rr = rs + cb + (c < ncol ? c : 0);
                gg[c] = gu[rr * 2 * Iw + i];
                uu[c] = gu[rr * 2 * Iw + Iw + i];
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                if (c >= ncol)  // uniform across the warp
                    break;
                const int64_t rr = rs + cb + c;
                const float g = gg[c], u = uu[c];
                // fast exponential and division: a few fp32 ulp, far below the bf16 rounding of
                // the gradients that follows
                const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
                const float act = g * sg;
                float ac = act, uc = u, ma = 1.0f, mu = 1.0f;
                if (L > 0.0f) {
                    if (act > L) {
                        ac = L;
                        ma = 0.0f;
                    }
                    if (u > L) {
                        uc = L;
                        mu = 0.0f;
                    } else if (u < -L) {
                        uc = -L;
                        mu = 0.0f;
                    }
                }
                const float dhu = v[c];
                if (!t.sh)
                    tr[lane * 17 + c] = ac * uc * dhu;  // this lane's term of h . dhu for column c
                const float dh = __shfl_sync(0xFFFFFFFFu, wl, c) * dhu;
                const float dg = dh * uc * ma * sg * (1.0f + g * (1.0f - sg));
                const float du = dh * ac * mu;
                dgu[rr * 2 * Iw + i] = __bfloat16_as_ushort(__float2bfloat16_rn(dg));
                dgu[rr * 2 * Iw + Iw + i] = __bfloat16_as_ushort(__float2bfloat16_rn(du));
            }
            if (!t.sh) {
                // dw of the block's columns: lane c sums column c of the warp's 32 feature
                // rows through the transpose buffer and adds it once (instead of a 5-step
                // shuffle reduction and an atomic per column)
                __syncwarp();
                if (lane < ncol) {
                    float sum = 0.0f;
#pragma unroll
                    for (int r = 0; r < 32; ++r)
                        sum += tr[r * 17 + lane];
                    atomicAdd(a.dw_pad + t.row0 + cb + lane, sum);
                }
                __syncwarp();
            }
        }
    } else if (MODE == kBwdDX) {
        const int64_t h = t.mb * 128 + row;
        for (int cb = 0; cb < t.ntok; cb += 32) {
            float v[32];
            tmem_load32(tq + cb, v);
            const int mycol = cb + lane;
            const int tok = mycol < t.ntok ? a.tok_pad[t.row0 + mycol] : 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int tk = __shfl_sync(0xFFFFFFFFu, tok, i);
                if (cb + i < t.ntok)
                    atomicAdd(a.dx + static_cast<int64_t>(tk) * a.H + h, v[i]);
            }
        }
    } else {
        // weight gradients: rows mb*128 + q*32 .. +32 of the output, columns nb*BN .. +BN, as
        // four 32 x 32 boxes. Lane l holds row l of a box: it writes its eight 16-byte pieces
        // in the 128-byte swizzle (piece j at j ^ (l % 8), conflict-free), and lane 0 stores
        // the box with one TMA copy. Two boxes alternate: a box is rewritten only after the
        // copy issued from it two boxes earlier has read it.
        const int64_t row0 = (MODE == kBwdWD ? (t.sh ? 0 : static_cast<int64_t>(t.g) * a.H)
                                             : (t.sh ? 0 : static_cast<int64_t>(t.g) * 2 * a.I)) +
                             t.mb * 128 + q * 32;
        uint8_t *stage = reinterpret_cast<uint8_t *>(tr);
        for (int cb = 0; cb < kBwdBN; cb += 32) {
            float v[32];
            tmem_load32(tq + cb, v);
            uint8_t *box = stage + ((cb >> 5) & 1) * kBwdEpiBox;
            if (lane == 0)
                bulk_wait_read<1>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float4 *dst = reinterpret_cast<float4 *>(box + lane * 128 + ((j ^ (lane & 7)) << 4));
                *dst = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_2d(om, box, t.nb * kBwdBN + cb, static_cast<int32_t>(row0));
                bulk_commit();
            }
        }
    }
}

// NSL = 64-wide K slices per stage (2: half as many stages of twice the size, so the MMA
// thread's barrier test and commit cover 8 MMAs; the tile's K must be a multiple of 128).
// Zeroes dW_gate_up[e] and dW_down[e] of every routed expert with no rows: each region is cut
// into kBwdZeroBytes pieces, CTA b stores pieces b, b + grid, ... from a zeroed shared-memory
// buffer with bulk copies (one issuing thread; the copies only read the constant buffer).
__device__ __forceinline__ void bwd_zero_untouched(const BwdArgs &a, const uint8_t *zero)
{
    const uint64_t gu_bytes = static_cast<uint64_t>(2) * a.I * a.H * 4, d_bytes = static_cast<uint64_t>(a.H) * a.I * 4;
    int issued = 0;
    for (int e = 0; e < a.E; ++e) {
        if (a.counts[e] != 0)
            continue;
        for (int r = 0; r < 2; ++r) {
            uint8_t *base = r == 0 ? reinterpret_cast<uint8_t *>(a.dWgu) + e * gu_bytes
                                   : reinterpret_cast<uint8_t *>(a.dWd) + e * d_bytes;
            const uint64_t bytes = r == 0 ? gu_bytes : d_bytes;
            for (uint64_t off = static_cast<uint64_t>(blockIdx.x) * kBwdZeroBytes; off < bytes;
                 off += static_cast<uint64_t>(gridDim.x) * kBwdZeroBytes) {
                const uint64_t n = bytes - off < kBwdZeroBytes ? bytes - off : kBwdZeroBytes;
                bulk_store(base + off, zero, static_cast<uint32_t>(n));
                if (++issued % 16 == 0)
                    bulk_commit();
            }
        }
    }
    bulk_commit();
    bulk_wait<0>();  // complete before the CTA (and its shared memory) goes away
}

template <int MODE, int NSL>
__global__ void __launch_bounds__(MODE == kBwdDH ? kBwdThreadsDH : kBwdThreads, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap a_r, const __grid_constant__ CUtensorMap a_s,
                    const __grid_constant__ CUtensorMap b_r, const __grid_constant__ CUtensorMap b_s,
                    const __grid_constant__ CUtensorMap o_r, const __grid_constant__ CUtensorMap o_s,
                    const BwdArgs a, const WaitCfg wc)
{
    constexpr bool kAmn = MODE != kBwdGU;
    constexpr bool kBmn = MODE == kBwdWD || MODE == kBwdWGU;
    // K slice: A, then B (MN-major 16 KB, or kBwdCap token rows of 128 bytes)
    constexpr uint32_t kSlice = kBwdTile + (kBmn ? kBwdTile : static_cast<uint32_t>(kBwdCap) * 128);
    constexpr uint32_t kStage = NSL * kSlice;
    constexpr int S = static_cast<int>(kBwdBarOff / kStage);
    static_assert(S >= 2 && S <= kBwdStages, "ring depth");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    uint8_t *smem = smem_raw + pad;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBwdBarOff);
    uint64_t *empty = full + S;
    uint64_t *accf = empty + S;
    uint64_t *acce = accf + 2;
    uint64_t *drain = acce + 2;
    uint32_t *holder = reinterpret_cast<uint32_t *>(smem + kBwdMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kBwdMiscOff + 4);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], MODE == kBwdDH ? kBwdDhEpiWarps : 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(holder, 2 * kBwdAcc);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *holder;
    const int tiles = bwd_tile_count<MODE>(a);

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_map(&a_r);
            tma_prefetch_map(&a_s);
            tma_prefetch_map(&b_r);
            tma_prefetch_map(&b_s);
            int it = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < tiles && !stop; tile += gridDim.x) {
                const BTile t = bwd_tile<MODE>(a, tile);
                // row-streaming modes: a chunk of at most 128 rows takes the 128-row token box
                const bool small = !kBmn && t.ntok <= 128;
                const CUtensorMap *mb = small ? (t.sh ? &o_s : &o_r) : (t.sh ? &b_s : &b_r);
                const uint32_t bbytes = kBmn ? kBwdTile : (small ? 128u : static_cast<uint32_t>(kBwdCap)) * 128u;
                for (int k0 = 0; k0 < t.K; k0 += 64 * NSL, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, wc, abort_flag)) {
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], NSL * (kBwdTile + bbytes));
                    for (int c = 0; c < NSL; ++c) {
                        uint8_t *A = smem + s * kStage + c * kSlice;
                        bwd_load<MODE>(a, t.sh ? &a_s : &a_r, mb, A, A + kBwdTile, &full[s], t, k0 + 64 * c);
                    }
                }
            }
            for (int i = it > S ? it - S : 0; i < it; ++i)
                mbar_wait_drain(&full[i % S], (i / S) & 1, wc);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tc = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
                const BTile t = bwd_tile<MODE>(a, tile);
                const int buf = tc & 1;
                if (!mbar_wait(&acce[buf], ((tc >> 1) & 1) ^ 1, wc, abort_flag))
                    break;
                tc_fence_after();
                const uint32_t d = tmem + buf * kBwdAcc;
                const uint32_t idesc = idesc_bf16_f32(128, (t.ntok + 15) & ~15) | (kAmn ? 1u << 15 : 0u) |
                                       (kBmn ? 1u << 16 : 0u);
                for (int k0 = 0; k0 < t.K; k0 += 64 * NSL, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(&full[s], (it / S) & 1, wc, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < NSL; ++c) {
                        const uint32_t sa = smem_u32(smem + s * kStage + c * kSlice);
                        const uint32_t sb = sa + kBwdTile;
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t ad =
                                kAmn ? sdesc_mn_sw128(sa + ks * 2048, 8192) : sdesc_kmajor_sw128(sa) + 2 * ks;
                            const uint64_t bd =
                                kBmn ? sdesc_mn_sw128(sb + ks * 2048, 8192) : sdesc_kmajor_sw128(sb) + 2 * ks;
                            umma_bf16(d, ad, bd, idesc, (k0 | c | ks) != 0);
                        }
                    }
                    umma_commit(&empty[s]);
                }
                if (ok)
                    umma_commit(&accf[buf]);
            }
            umma_commit(drain);
            mbar_wait_drain(drain, 0, wc);
        }
    } else if (MODE == kBwdDH && warp == 2 + kBwdDhEpiWarps) {
        // DH only: zero the gradients of untouched experts
        uint8_t *zero = smem + kBwdZeroOff;
        for (uint32_t i = lane * 16; i < kBwdZeroBytes; i += 32 * 16)
            *reinterpret_cast<uint4 *>(zero + i) = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0)
            bwd_zero_untouched(a, zero);
        __syncwarp();
    } else {
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;  // DH: which of the lane quarter's two warps
        float *tr = reinterpret_cast<float *>(smem + kBwdEpiOff +
                                              (MODE == kBwdDH ? (warp - 2) * kBwdDhTr : q * kBwdEpiWarp));
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            const BTile t = bwd_tile<MODE>(a, tile);
            const int buf = tc & 1;
            if (!warp_wait(&accf[buf], (tc >> 1) & 1, wc, abort_flag))
                break;
            tc_fence_after();
            bwd_epilogue<MODE>(a, tmem + buf * kBwdAcc, t, q, half, lane, tr, t.sh ? &o_s : &o_r);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acce[buf]);
        }
        if (lane == 0)
            bulk_wait<0>();  // this warp's gradient stores have completed before the CTA exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kBwdAcc);
    }
}

template <int MODE, int NSL>
cudaError_t launch_mode(const CUtensorMap &a_r, const CUtensorMap &a_s, const CUtensorMap &b_r, const CUtensorMap &b_s,
                        const CUtensorMap &o_r, const CUtensorMap &o_s, const BwdArgs &a, const WaitCfg &wc, int grid,
                        cudaStream_t stream)
{
    cudaError_t err = cudaFuncSetAttribute(bwd_gemm_kernel<MODE, NSL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kBwdSmem));
    if (err != cudaSuccess)
        return err;
    const int threads = MODE == kBwdDH ? kBwdThreadsDH : kBwdThreads;
    bwd_gemm_kernel<MODE, NSL><<<grid, threads, kBwdSmem, stream>>>(a_r, a_s, b_r, b_s, o_r, o_s, a, wc);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_gemm(int mode, const CUtensorMap &a_r, const CUtensorMap &a_s, const CUtensorMap &b_r,
                            const CUtensorMap &b_s, const CUtensorMap &o_r, const CUtensorMap &o_s, const BwdArgs &a,
                            const WaitCfg &wc, int grid, cudaStream_t stream)
{
    // row-streaming modes: one K slice per stage (48 KB stages, four deep); the
    // weight-gradient modes reduce over 64-row padded groups (32 KB stages, six deep)
    switch (mode) {
    case kBwdGU:
        return launch_mode<kBwdGU, 1>(a_r, a_s, b_r, b_s, o_r, o_s, a, wc, grid, stream);
    case kBwdDH:
        return launch_mode<kBwdDH, 1>(a_r, a_s, b_r, b_s, o_r, o_s, a, wc, grid, stream);
    case kBwdDX:
        return launch_mode<kBwdDX, 1>(a_r, a_s, b_r, b_s, o_r, o_s, a, wc, grid, stream);
    case kBwdWD:
        return launch_mode<kBwdWD, 1>(a_r, a_s, b_r, b_s, o_r, o_s, a, wc, grid, stream);
    case kBwdWGU:
        return launch_mode<kBwdWGU, 1>(a_r, a_s, b_r, b_s, o_r, o_s, a, wc, grid, stream);
    default:
        return cudaErrorInvalidValue;
    }
}

}  // namespace moe
